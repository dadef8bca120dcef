// H (+)= 2 X^T X on the tensor cores (tutorial "阶段一", H = 2 X^T X).
// X (n x d_in, row-major) is first transposed to X^T (d_in x n_pad, zero padded) so
// both GEMM operands are K-major; for fp32 X the transpose also splits each value
// into two tf32 parts for the 3xTF32 product.  Only tiles on or above the diagonal
// are computed; each off-diagonal tile is also written to its mirror position.
#pragma once
#include "gemm_tc.cuh"

namespace gq {

constexpr int kHessNPad = 64;

// 64x64 tiled transpose: XT[c, t] = X[t, c] for t < n, 0 for n <= t < n_pad.  Both global
// sides move 16-byte vectors (8 bf16) with a warp covering four whole 128-byte rows; the
// shared tile [t][c] has 33-word rows, so the row-wise writes are conflict-free and the
// column-wise reads at most 2-way.  d_in % 8 == 0 and n_pad % 64 == 0.
constexpr int TR_T = 64, TR_C = 64, TR_LD = TR_C + 2;
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const uint16_t* __restrict__ X, long long n,
                                                             long long d_in, long long n_pad,
                                                             uint16_t* __restrict__ XT) {
    __shared__ __align__(16) uint16_t tile[TR_T][TR_LD];   // tile[t][c]
    const long long t0 = (long long)blockIdx.x * TR_T, c0 = (long long)blockIdx.y * TR_C;
    for (int e = threadIdx.x; e < TR_T * (TR_C / 8); e += blockDim.x) {
        const int r = e >> 3, v8 = e & 7;
        const long long t = t0 + r, c = c0 + 8 * v8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (t < n && c < d_in) v = *reinterpret_cast<const uint4*>(X + t * d_in + c);
        uint32_t* dst = reinterpret_cast<uint32_t*>(&tile[r][8 * v8]);
        dst[0] = v.x;
        dst[1] = v.y;
        dst[2] = v.z;
        dst[3] = v.w;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < TR_C * (TR_T / 8); e += blockDim.x) {
        const int cr = e >> 3, v8 = e & 7;
        const long long c = c0 + cr, t = t0 + 8 * v8;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            w[q] = (uint32_t)tile[8 * v8 + 2 * q][cr] | ((uint32_t)tile[8 * v8 + 2 * q + 1][cr] << 16);
        if (c < d_in && t < n_pad) *reinterpret_cast<uint4*>(XT + c * n_pad + t) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__global__ void transpose_split_f32_kernel(const float* __restrict__ X, long long n, long long d_in,
                                           long long n_pad, float* __restrict__ XT_hi,
                                           float* __restrict__ XT_lo) {
    __shared__ float tile[32][33];
    const long long t0 = (long long)blockIdx.x * 32, c0 = (long long)blockIdx.y * 32;
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const long long t = t0 + r, c = c0 + threadIdx.x;
        tile[r][threadIdx.x] = (t < n && c < d_in) ? X[t * d_in + c] : 0.f;
    }
    __syncthreads();
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const long long c = c0 + r, t = t0 + threadIdx.x;
        if (c < d_in && t < n_pad) {
            float hi, lo;
            split_tf32(tile[threadIdx.x][r], hi, lo);
            XT_hi[c * n_pad + t] = hi;
            XT_lo[c * n_pad + t] = lo;
        }
    }
}

}  // namespace gq

namespace gqh {

inline long long hess_npad(long long n) { return (n + gq::kHessNPad - 1) / gq::kHessNPad * gq::kHessNPad; }

inline size_t hessian_ws_bytes(long long n, long long d_in, gptq_dtype xt) {
    const long long np = hess_npad(n);
    return xt == GPTQ_BF16 ? (size_t)(d_in * np * 2) : (size_t)(2 * d_in * np * 4);
}

// Both Hessian entry points run this: the workspace one (no_alloc = false) and the
// fixed-scratch one (no_alloc = true: ws is the library's static scratch array, and no
// host-side bookkeeping that allocates is used), so they launch the same kernels with the
// same segmented accumulation.
inline cudaError_t hessian_run(const void* X, gptq_dtype xt, long long n, long long d_in, float* H,
                               int accumulate, void* ws, cudaStream_t st, bool no_alloc = false) {
    const char* tname = no_alloc ? nullptr : "transpose_x";
    const long long np = hess_npad(n);
    dim3 tb(32, 8);
    dim3 grid((unsigned)(np / 32), (unsigned)((d_in + 31) / 32));
    const dim3 grid64((unsigned)(np / gq::TR_T), (unsigned)((d_in + gq::TR_C - 1) / gq::TR_C));
    gq::GemmArgs p = gemm_args((int)d_in, (int)d_in, (int)np);
    p.triangular = 1;
    p.mirror = 1;
    p.alpha = 2.f;
    p.beta = accumulate ? 1.f : 0.f;
    p.write_c = 1;
    EpiMats o;
    o.c = Mat{H, (uint64_t)d_in, (uint64_t)d_in, (uint64_t)d_in};
    if (xt == GPTQ_BF16) {
        uint16_t* XT = static_cast<uint16_t*>(ws);
        {
            gqh::TimedScope ts__(tname, st);
            gq::transpose_bf16_kernel<<<grid64, 256, 0, st>>>(static_cast<const uint16_t*>(X), n, d_in, np, XT);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        Mat m{XT, (uint64_t)d_in, (uint64_t)np, (uint64_t)np};
        return launch_gemm<gq::KIND_BF16, 4, 128, 16>(m, m, m, m, o, p, 1, st, "hessian_syrk", 0, false, no_alloc);
    }
    float* hi = static_cast<float*>(ws);
    float* lo = hi + d_in * np;
    {
        gqh::TimedScope ts__(tname, st);
        gq::transpose_split_f32_kernel<<<grid, tb, 0, st>>>(static_cast<const float*>(X), n, d_in, np, hi, lo);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    Mat mh{hi, (uint64_t)d_in, (uint64_t)np, (uint64_t)np};
    Mat ml{lo, (uint64_t)d_in, (uint64_t)np, (uint64_t)np};
    return launch_gemm<gq::KIND_TF32X3, 2, 128, 4>(mh, ml, mh, ml, o, p, 1, st, "hessian_syrk", 0, false,
                                                   no_alloc);
}

}  // namespace gqh
