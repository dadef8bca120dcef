// Activation ordering ("激活排序（desc_act）" on the GPTQ tutorial page): the columns
// are visited in an order ranked by the sum of absolute input activations.  The
// factorization and the column loop run unchanged on the permuted problem
// Hp[i][j] = H[perm[i]][perm[j]], Wp[:, k] = W[:, perm[k]]; the packed codes are then
// put back in the original column order and a per-column group index is written.
//
// Kernels here: the activation statistic, the ranking, the gathers, and the repack.
// Every kernel that reads a caller's permutation checks each entry against d and
// records GPTQ_ERR_INVALID_ARG (the entry's position) instead of reading out of range.
#pragma once
#include "common.cuh"
#include "pack.cuh"

namespace gq {

constexpr int AS_COLS = 64;        // columns per CTA of act_sum_kernel (8 lanes x 8 columns)
constexpr int AS_ROWS = 32;        // rows in flight per pass (256 threads / 8 lanes)
constexpr int RK_THREADS = 256;    // columns ranked per CTA
constexpr int RK_CHUNK = 256;      // keys compared per CTA (one shared-memory tile)

// a[c] (+)= sum_t |X[t, c]| in fp64.  Thread (ty, tx) owns columns c0 + 8 tx .. + 7 of
// rows ty, ty + 32, ...; the 32 partial sums per column are added in a fixed order, so
// the result does not depend on scheduling.  d % 8 == 0.  A non-finite sum is reported.
template <bool BF16>
__global__ void __launch_bounds__(256) act_sum_kernel(const void* __restrict__ Xv, long long n, long long d,
                                                      int accumulate, double* __restrict__ a) {
    __shared__ double part[AS_ROWS][AS_COLS + 1];
    const int tx = threadIdx.x & 7, ty = threadIdx.x >> 3;
    const long long c0 = (long long)blockIdx.x * AS_COLS + tx * 8;
    double s[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (c0 < d) {
        for (long long r = ty; r < n; r += AS_ROWS) {
            float v[8];
            if (BF16) {
                const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(Xv) + r * d + c0);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    v[2 * q] = __uint_as_float(w[q] << 16);
                    v[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
                }
            } else {
                const float* p = static_cast<const float*>(Xv) + r * d + c0;
                const float4 x0 = *reinterpret_cast<const float4*>(p);
                const float4 x1 = *reinterpret_cast<const float4*>(p + 4);
                v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
                v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) s[q] += (double)fabsf(v[q]);
        }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) part[ty][tx * 8 + q] = s[q];
    __syncthreads();
    if (threadIdx.x < AS_COLS) {
        const long long c = (long long)blockIdx.x * AS_COLS + threadIdx.x;
        if (c < d) {
            double t = 0.0;
            for (int i = 0; i < AS_ROWS; ++i) t += part[i][threadIdx.x];
            const double out = accumulate ? a[c] + t : t;
            if (!isfinite(out)) record_status(GPTQ_ERR_NONFINITE, c);
            a[c] = out;
        }
    }
}

// Total order on doubles as unsigned integers (both zeros equal); ``descending``
// flips it.  NaN sorts by its bit pattern.
__device__ __forceinline__ unsigned long long order_key(double x, int descending) {
    if (x == 0.0) x = 0.0;
    const unsigned long long b = (unsigned long long)__double_as_longlong(x);
    const unsigned long long k = (b >> 63) ? ~b : (b | 0x8000000000000000ull);
    return descending ? ~k : k;
}

// rank[c] += #{j in this CTA's key chunk : key_j < key_c, or key_j == key_c and j < c}.
// Grid (ceil(d / 256), ceil(d / 256)); rank must be zero before the launch.  Integer
// atomics make the sum order-independent.
__global__ void __launch_bounds__(RK_THREADS) act_rank_kernel(const double* __restrict__ a, long long d,
                                                              int descending, int* __restrict__ rank) {
    __shared__ unsigned long long keys[RK_CHUNK];
    const long long j0 = (long long)blockIdx.y * RK_CHUNK;
    const int nj = (int)(d - j0 < RK_CHUNK ? d - j0 : RK_CHUNK);
    for (int i = threadIdx.x; i < nj; i += blockDim.x) keys[i] = order_key(a[j0 + i], descending);
    __syncthreads();
    const long long c = (long long)blockIdx.x * RK_THREADS + threadIdx.x;
    if (c >= d) return;
    const unsigned long long kc = order_key(a[c], descending);
    int cnt = 0;
    for (int i = 0; i < nj; ++i) {
        const unsigned long long kj = keys[i];
        cnt += (kj < kc) || (kj == kc && j0 + i < c);
    }
    if (cnt) atomicAdd(rank + c, cnt);
}

// perm[rank[c]] = c.
__global__ void act_perm_kernel(const int* __restrict__ rank, long long d, int* __restrict__ perm) {
    for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < d; c += (long long)gridDim.x * blockDim.x)
        perm[rank[c]] = (int)c;
}

// rank[perm[k]] = k for a caller's permutation; rank must be -1 everywhere before the
// launch.  An entry out of [0, d) or a repeated entry is recorded (its position k).
__global__ void perm_invert_kernel(const int* __restrict__ perm, long long d, int* __restrict__ rank) {
    for (long long k = blockIdx.x * (long long)blockDim.x + threadIdx.x; k < d; k += (long long)gridDim.x * blockDim.x) {
        const int c = perm[k];
        if (c < 0 || c >= d) {
            record_status(GPTQ_ERR_INVALID_ARG, k);
            continue;
        }
        if (atomicExch(rank + c, (int)k) != -1) record_status(GPTQ_ERR_INVALID_ARG, k);
    }
}

__device__ __forceinline__ int checked_index(const int* __restrict__ perm, long long k, long long d) {
    const int c = perm[k];
    if (c < 0 || c >= d) {
        record_status(GPTQ_ERR_INVALID_ARG, k);
        return 0;
    }
    return c;
}

// Wp[o][k] = W[o][perm[k]] with the row staged in shared memory: 16-byte loads of the
// row, gathers from shared memory, 16-byte stores (d_in % 8 == 0; d_in * 4 bytes of
// dynamic shared memory).  One CTA per row, rows strided over the grid.
__global__ void __launch_bounds__(256) gather_cols_smem_kernel(const float* __restrict__ W,
                                                               const int* __restrict__ perm, long long d_out,
                                                               long long d_in, float* __restrict__ Wp) {
    extern __shared__ float4 row4[];
    const float* row = reinterpret_cast<const float*>(row4);
    const long long q4 = d_in / 4;
    for (long long o = blockIdx.x; o < d_out; o += gridDim.x) {
        const float4* src = reinterpret_cast<const float4*>(W + o * d_in);
        for (long long k = threadIdx.x; k < q4; k += blockDim.x) row4[k] = src[k];
        __syncthreads();
        float4* dst = reinterpret_cast<float4*>(Wp + o * d_in);
        for (long long k = threadIdx.x; k < q4; k += blockDim.x) {
            float4 v;
            v.x = row[checked_index(perm, 4 * k, d_in)];
            v.y = row[checked_index(perm, 4 * k + 1, d_in)];
            v.z = row[checked_index(perm, 4 * k + 2, d_in)];
            v.w = row[checked_index(perm, 4 * k + 3, d_in)];
            dst[k] = v;
        }
        __syncthreads();
    }
}

// Wp[o][k] = W[o][perm[k]] for rows too wide for shared memory: one CTA per row, the
// gathered reads go through L1.
__global__ void __launch_bounds__(256) gather_cols_kernel(const float* __restrict__ W, const int* __restrict__ perm,
                                                          long long d_out, long long d_in, float* __restrict__ Wp) {
    for (long long o = blockIdx.x; o < d_out; o += gridDim.x) {
        const float* src = W + o * d_in;
        float* dst = Wp + o * d_in;
        for (long long k = threadIdx.x; k < d_in; k += blockDim.x) dst[k] = src[checked_index(perm, k, d_in)];
    }
}

// Repack the codes of the permuted column loop (qweight layout, code k of row o =
// column perm[k]) in the original column order: code c of row o = code rank[c] of the
// permuted stream.  One thread per output word, consecutive threads on consecutive
// rows of one word index, so the reads of one code position are coalesced.  Threads
// with idx < d_in also write g_idx[idx] = rank[idx] / g.
__global__ void unpermute_codes_kernel(const int32_t* __restrict__ qw_perm, const int* __restrict__ rank,
                                       long long d_out, long long d_in, int bits, int g,
                                       int32_t* __restrict__ qweight, int32_t* __restrict__ g_idx) {
    const long long nwords = (d_in * bits + 31) / 32;
    const long long total = nwords * d_out;
    const uint32_t mask = (1u << bits) - 1u;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < max(total, d_in);
         idx += (long long)gridDim.x * blockDim.x) {
        if (idx < d_in) g_idx[idx] = max(rank[idx], 0) / g;
        if (idx >= total) continue;
        const long long k = idx / d_out, o = idx % d_out;
        const long long bit0 = k * 32;
        const long long j0 = bit0 / bits;
        const long long j1 = min(d_in - 1, (bit0 + 31) / bits);
        unsigned long long acc = 0;
        for (long long j = j0; j <= j1; ++j) {
            const int r = rank[j];   // -1 only after an invalid permutation (already recorded)
            const uint32_t q = stream_code(qw_perm + o, d_out, r < 0 ? 0 : r, bits) & mask;
            acc |= (unsigned long long)q << (j * bits - bit0 + 8);   // >= 6: a code starts at most 2 bits early
        }
        qweight[k * d_out + o] = (int32_t)(uint32_t)(acc >> 8);
    }
}

}  // namespace gq
