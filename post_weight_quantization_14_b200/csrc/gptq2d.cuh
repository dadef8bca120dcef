// GPTQ-2D: two-sided adaptive rounding of a real matrix X (m x n) to an integer matrix Z
// under the quadratic metric tr((X - Z)^T G_left (X - Z) G_right) (GPTQ-2D summary, "方法"
// and "核心洞察").  Inputs are the upper Cholesky factors U_left of G_left^-1 and U_right
// of G_right^-1; the Kronecker factor U_right (x) U_left is never formed.
//
// The entries are taken anti-diagonal by anti-diagonal (i + j = k, k = 0 .. m + n - 2).
// The errors of entry (i', j') reach (i, j) only when i' <= i and j' <= j, so the entries
// of one anti-diagonal do not depend on one another and are rounded in parallel, one warp
// each, from the state left by the earlier anti-diagonals:
//   v_ij = X_ij - sum_{r <= i} U_left[r, i] T[r, j]      (a warp-wide dot product)
//   Z_ij = rint(v_ij),  e_ij = (v_ij - Z_ij) / (U_left[i, i] U_right[j, j])
//   T[i, j'] += e_ij U_right[j, j']  for j' >= j          (row i only: no conflicts)
// with T[i, :] the running sum of the pushed-forward errors of row i.  fp64 throughout,
// round half to even, no clamp (the unbounded integer lattice).  One CTA per problem of a
// batch; T in shared memory when it fits, else in the workspace; U_left is read
// transposed (a copy in the workspace) so the dot products read contiguous memory.
#pragma once
#include "common.cuh"

namespace gq {

constexpr int G2_THREADS = 1024;
constexpr long long G2_SMEM_T_MAX = 160 * 1024;   // bytes of T kept in shared memory

// ULT[i][r] = U_left[r][i]
__global__ void g2_transpose_kernel(const double* __restrict__ UL, long long m, double* __restrict__ ULT) {
    __shared__ double tile[32][33];
    const long long r0 = (long long)blockIdx.y * 32, c0 = (long long)blockIdx.x * 32;
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const long long rr = r0 + r, cc = c0 + threadIdx.x;
        tile[r][threadIdx.x] = (rr < m && cc < m) ? UL[rr * m + cc] : 0.0;
    }
    __syncthreads();
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const long long rr = c0 + r, cc = r0 + threadIdx.x;
        if (rr < m && cc < m) ULT[rr * m + cc] = tile[threadIdx.x][r];
    }
}

__global__ void __launch_bounds__(G2_THREADS)
    gptq2d_kernel(const double* __restrict__ X, int m, int n, const double* __restrict__ ULT,
                  const double* __restrict__ UR, int32_t* __restrict__ Z, double* __restrict__ T_ws, int t_smem) {
    extern __shared__ double g2_smem[];
    constexpr unsigned FULL = 0xffffffffu;
    const long long b = blockIdx.x;
    const long long mn = (long long)m * n;
    const double* Xb = X + b * mn;
    int32_t* Zb = Z + b * mn;
    double* T = t_smem ? g2_smem : T_ws + b * mn;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
    for (long long e = tid; e < mn; e += blockDim.x) T[e] = 0.0;
    __syncthreads();
    for (int k = 0; k < m + n - 1; ++k) {
        const int i0 = max(0, k - n + 1), i1 = min(m - 1, k);
        for (int i = i0 + warp; i <= i1; i += nw) {
            const int j = k - i;
            const double* ul = ULT + (long long)i * m;   // column i of U_left
            double acc = 0.0;
            for (int r = lane; r <= i; r += 32) acc = fma(ul[r], T[(long long)r * n + j], acc);
#pragma unroll
            for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
            const double v = Xb[(long long)i * n + j] - acc;
            const double z = rint(v);
            const double err = (v - z) / (ul[i] * UR[(long long)j * n + j]);
            if (lane == 0) {
                if (!isfinite(v) || fabs(z) > 2147483647.0) {
                    record_status(GPTQ_ERR_NONFINITE, b * mn + (long long)i * n + j);
                    Zb[(long long)i * n + j] = 0;
                } else {
                    Zb[(long long)i * n + j] = (int32_t)z;
                }
            }
            const double* ur = UR + (long long)j * n;
            double* t = T + (long long)i * n;
            for (int jj = j + lane; jj < n; jj += 32) t[jj] = fma(err, ur[jj], t[jj]);
        }
        __syncthreads();
    }
}

}  // namespace gq

namespace gqh {

inline bool g2_t_in_smem(long long m, long long n) { return m * n * 8 <= gq::G2_SMEM_T_MAX; }

inline size_t g2_ws_bytes(long long m, long long n, long long batch) {
    size_t b = (size_t)(m * m * 8 + 255) / 256 * 256;   // U_left transposed
    if (!g2_t_in_smem(m, n)) b += (size_t)(batch * m * n * 8);
    return b;
}

inline cudaError_t g2_run(const double* X, long long m, long long n, long long batch, const double* UL,
                          const double* UR, int32_t* Z, void* ws, cudaStream_t st) {
    double* ULT = static_cast<double*>(ws);
    double* T = reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + (size_t)(m * m * 8 + 255) / 256 * 256);
    {
        gqh::TimedScope ts__("g2_transpose", st);
        const dim3 grid((unsigned)((m + 31) / 32), (unsigned)((m + 31) / 32));
        gq::g2_transpose_kernel<<<grid, dim3(32, 8), 0, st>>>(UL, m, ULT);
    }
    GQ_TRY(cudaGetLastError());
    const bool in_smem = g2_t_in_smem(m, n);
    const int smem = in_smem ? (int)(m * n * 8) : 0;
    if (smem > 48 * 1024) GQ_TRY(ensure_smem_attr(reinterpret_cast<const void*>(gq::gptq2d_kernel), smem));
    {
        gqh::TimedScope ts__("gptq2d", st);
        gq::gptq2d_kernel<<<(unsigned)batch, gq::G2_THREADS, (size_t)smem, st>>>(X, (int)m, (int)n, ULT, UR, Z, T,
                                                                               in_smem ? 1 : 0);
    }
    return cudaGetLastError();
}

}  // namespace gqh
