// Layer output error E = ||(W - W_hat) X^T||_F^2 (tutorial "阶段一": the squared error of
// the layer's outputs over the calibration tokens, the quantity GPTQ minimises), with its
// per-row parts.
//
// D = W - W_hat and X are split into bf16 pairs (x ~ hi + lo, 16 significant bits), the
// product Y = D X^T [d_out x n] runs on the tensor cores as three bf16 products (hi hi,
// hi lo, lo hi) with fp32 accumulation in segments, and each row's sum of Y^2 is taken in
// fp64 by one warp; the total adds the rows in a fixed order (one CTA, fixed tree), so the
// result has the same bits on every run.
#pragma once
#include "gemm_tc.cuh"

namespace gq {

// D = W - W_hat as bf16 split bit patterns; four elements per thread step (n4 = elements / 4).
__global__ void loss_diff_split_kernel(const float4* __restrict__ W, const float4* __restrict__ Wh, long long n4,
                                       uint2* __restrict__ D_hi, uint2* __restrict__ D_lo) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
        const float4 a = W[i], b = Wh[i];
        const float d[4] = {a.x - b.x, a.y - b.y, a.z - b.z, a.w - b.w};
        uint16_t h[4], l[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) split_bf16(d[q], h[q], l[q]);
        D_hi[i] = make_uint2((uint32_t)h[0] | ((uint32_t)h[1] << 16), (uint32_t)h[2] | ((uint32_t)h[3] << 16));
        D_lo[i] = make_uint2((uint32_t)l[0] | ((uint32_t)l[1] << 16), (uint32_t)l[2] | ((uint32_t)l[3] << 16));
    }
}

// X as bf16 split bit patterns: a bf16 X is its own hi part (lo = 0); an fp32 X is split.
__global__ void loss_x_split_kernel(const void* __restrict__ X, int is_bf16, long long n4, uint2* __restrict__ X_hi,
                                    uint2* __restrict__ X_lo) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
        if (is_bf16) {
            X_hi[i] = reinterpret_cast<const uint2*>(X)[i];
            X_lo[i] = make_uint2(0u, 0u);
        } else {
            const float4 a = reinterpret_cast<const float4*>(X)[i];
            const float v[4] = {a.x, a.y, a.z, a.w};
            uint16_t h[4], l[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) split_bf16(v[q], h[q], l[q]);
            X_hi[i] = make_uint2((uint32_t)h[0] | ((uint32_t)h[1] << 16), (uint32_t)h[2] | ((uint32_t)h[3] << 16));
            X_lo[i] = make_uint2((uint32_t)l[0] | ((uint32_t)l[1] << 16), (uint32_t)l[2] | ((uint32_t)l[3] << 16));
        }
    }
}

// row_loss[o] = sum_t Y[o, t]^2 in fp64, one warp per row (lanes stride the row, then a
// fixed shuffle tree).
__global__ void loss_row_sumsq_kernel(const float* __restrict__ Y, long long d_out, long long n, long long ldy,
                                      double* __restrict__ row_loss) {
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= d_out) return;
    const float* y = Y + row * ldy;
    double acc = 0.0;
    for (long long t = lane; t < n; t += 32) {
        const double v = (double)y[t];
        acc = fma(v, v, acc);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) row_loss[row] = acc;
}

// *loss = sum of row_loss[0 .. d_out) in a fixed order (one CTA of LOSS_SUM_THREADS).
constexpr int LOSS_SUM_THREADS = 1024;
__global__ void __launch_bounds__(LOSS_SUM_THREADS) loss_total_kernel(const double* __restrict__ row_loss,
                                                                     long long d_out, double* __restrict__ loss) {
    __shared__ double part[LOSS_SUM_THREADS];
    double acc = 0.0;
    for (long long i = threadIdx.x; i < d_out; i += LOSS_SUM_THREADS) acc += row_loss[i];
    part[threadIdx.x] = acc;
    __syncthreads();
    for (int s = LOSS_SUM_THREADS / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) part[threadIdx.x] += part[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) *loss = part[0];
}

}  // namespace gq

namespace gqh {

inline size_t loss_align(size_t b) { return (b + 255) / 256 * 256; }
inline long long loss_ldy(long long n) { return (n + 3) / 4 * 4; }

// Workspace: D split (2 x d_out x d_in bf16), X split (2 x n x d_in bf16), Y (d_out x ldy
// fp32), row losses (d_out fp64).
inline size_t loss_ws_bytes(long long d_out, long long d_in, long long n) {
    return 2 * loss_align((size_t)(d_out * d_in * 2)) + 2 * loss_align((size_t)(n * d_in * 2)) +
           loss_align((size_t)(d_out * loss_ldy(n) * 4)) + loss_align((size_t)(d_out * 8));
}

inline cudaError_t loss_run(const float* W, const float* Wh, const void* X, bool x_bf16, long long d_out,
                            long long d_in, long long n, double* row_loss, double* loss, void* ws, cudaStream_t st) {
    uint8_t* p = static_cast<uint8_t*>(ws);
    uint16_t* D_hi = reinterpret_cast<uint16_t*>(p);
    p += loss_align((size_t)(d_out * d_in * 2));
    uint16_t* D_lo = reinterpret_cast<uint16_t*>(p);
    p += loss_align((size_t)(d_out * d_in * 2));
    uint16_t* X_hi = reinterpret_cast<uint16_t*>(p);
    p += loss_align((size_t)(n * d_in * 2));
    uint16_t* X_lo = reinterpret_cast<uint16_t*>(p);
    p += loss_align((size_t)(n * d_in * 2));
    float* Y = reinterpret_cast<float*>(p);
    p += loss_align((size_t)(d_out * loss_ldy(n) * 4));
    double* rows = row_loss ? row_loss : reinterpret_cast<double*>(p);
    const int sms = num_sms();
    {
        TimedScope ts__("loss_split", st);
        gq::loss_diff_split_kernel<<<4 * sms, 256, 0, st>>>(reinterpret_cast<const float4*>(W),
                                                             reinterpret_cast<const float4*>(Wh), d_out * d_in / 4,
                                                             reinterpret_cast<uint2*>(D_hi), reinterpret_cast<uint2*>(D_lo));
        gq::loss_x_split_kernel<<<4 * sms, 256, 0, st>>>(X, x_bf16 ? 1 : 0, n * d_in / 4, reinterpret_cast<uint2*>(X_hi),
                                                          reinterpret_cast<uint2*>(X_lo));
    }
    GQ_TRY(cudaGetLastError());
    const long long ldy = loss_ldy(n);
    Mat dh{D_hi, (uint64_t)d_out, (uint64_t)d_in, (uint64_t)d_in};
    Mat dl{D_lo, (uint64_t)d_out, (uint64_t)d_in, (uint64_t)d_in};
    Mat xh{X_hi, (uint64_t)n, (uint64_t)d_in, (uint64_t)d_in};
    Mat xl{X_lo, (uint64_t)n, (uint64_t)d_in, (uint64_t)d_in};
    EpiMats o;
    o.c = Mat{Y, (uint64_t)d_out, (uint64_t)n, (uint64_t)ldy};
    gq::GemmArgs g = gemm_args((int)d_out, (int)n, (int)d_in);
    g.write_c = 1;
    GQ_TRY((launch_gemm<gq::KIND_BF16X3, 2, 128, 8>(dh, dl, xh, xl, o, g, 1, st, "loss_gemm", 0, true)));
    {
        TimedScope ts__("loss_reduce", st);
        gq::loss_row_sumsq_kernel<<<(unsigned)((d_out + 7) / 8), 256, 0, st>>>(Y, d_out, n, ldy, rows);
        gq::loss_total_kernel<<<1, gq::LOSS_SUM_THREADS, 0, st>>>(rows, d_out, loss);
    }
    return cudaGetLastError();
}

}  // namespace gqh
