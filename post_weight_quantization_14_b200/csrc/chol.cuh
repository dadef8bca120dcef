// U = upper Cholesky factor of Hd^-1, Hd = H + lambda I  (tutorial "阶段一": damping,
// Cholesky factor, upper triangular, read as the factor of the inverse Hessian).
//
// Route: Hd = R R^T with R upper triangular (Cholesky started from the bottom-right
// corner), then U = R^-1; U is upper with U^T U = R^-T R^-1 = Hd^-1, which is the
// unique upper Cholesky factor of Hd^-1.
//
// Blocked by NB = 128 on n = roundup(d, 128) (padding rows/columns get an identity
// diagonal, which leaves the leading d x d block of U unchanged):
//   for j = T-1 .. 0:
//     leaf(j):   R_jj = UL-Cholesky(A_jj), X_jj = R_jj^-1           (one CTA, fp32)
//     panel(j):  R_{0:j, j} = A_{0:j, j} X_jj^T                      (3xTF32 tcgen05)
//     update(j): A_{0:j, 0:j} -= R_{0:j, j} R_{0:j, j}^T             (3xTF32 tcgen05)
//   then U = R^-1 by doubling: for s = 128, 256, ...: for each diagonal pair
//     [[R_a, B], [0, R_c]] with known inverses U_a, U_c:  U_b = -U_a (B U_c).
#pragma once
#include "gemm_tc.cuh"

namespace gq {

constexpr int NB = 128;

// lambda = damp_rel * mean(diag H), accumulated in double.
__global__ void diag_mean_kernel(const float* __restrict__ H, long long d, float damp_rel,
                                 float* __restrict__ lam_out) {
    __shared__ double part[32];
    double s = 0.0;
    for (long long i = threadIdx.x; i < d; i += blockDim.x) s += (double)H[i * d + i];
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += part[w];
        const double mean = t / (double)d;
        if (!isfinite(mean)) record_status(GPTQ_ERR_NONFINITE, -1);
        else if (!(mean > 0.0)) record_status(GPTQ_ERR_INVALID_ARG, -1);
        lam_out[0] = (float)(damp_rel * mean);
    }
}

// A (n x n) = Hd with only the upper triangle of H read; padding gets identity.
__global__ void damp_copy_kernel(const float* __restrict__ H, long long d, long long n,
                                 const float* __restrict__ lam, float* __restrict__ A) {
    __shared__ float tile[32][33];
    const long long bi = blockIdx.y, bj = blockIdx.x;
    const bool lower = bi > bj;
    const long long si = lower ? bj : bi, sj = lower ? bi : bj;  // source tile (upper)
    const float l = lam[0];
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const long long i = si * 32 + r, j = sj * 32 + threadIdx.x;
        float v = 0.f;
        if (i < d && j < d) {
            v = H[i * d + j];
            if (i <= j && !isfinite(v)) record_status(GPTQ_ERR_NONFINITE, i * d + j);
        }
        tile[r][threadIdx.x] = v;
    }
    __syncthreads();
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const long long i = bi * 32 + r, j = bj * 32 + threadIdx.x;
        if (i >= n || j >= n) continue;
        float v = lower ? tile[threadIdx.x][r] : tile[r][threadIdx.x];
        if (i == j) v = (i < d) ? v + l : 1.f;
        A[i * n + j] = v;
    }
}

// Split A[0:rows, col0:col0+128] into tf32 hi/lo arrays with leading dimension 128.
__global__ void split_panel_kernel(const float* __restrict__ A, long long n, int rows, int col0,
                                   float* __restrict__ hi, float* __restrict__ lo) {
    const long long total = (long long)rows * NB;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const long long r = e >> 7, c = e & 127;
        float h, l;
        split_tf32(A[r * n + col0 + c], h, l);
        hi[e] = h;
        lo[e] = l;
    }
}

// Zero the strictly-lower 128-blocks of the d x d output U (diagonal blocks are
// written in full by the leaf kernel).
__global__ void zero_lower_blocks_kernel(float* __restrict__ U, long long d) {
    const long long total = d * d;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const long long r = e / d, c = e % d;
        if ((r >> 7) > (c >> 7)) U[e] = 0.f;
    }
}

// Leaf: factor and invert one 128x128 diagonal block of A in shared memory.
// Writes X = R_jj^-1 (upper, zeros below the diagonal) to the public U (clipped to
// d), its row-major tf32 split (U_hi/U_lo) and its transposed split (UT_hi/UT_lo).
struct LeafSmem {
    float a[NB][NB + 1];
    float u[NB][NB + 1];
    float xinv[4][32][33];
    float tmp[3][32][33];
};

__global__ void __launch_bounds__(512, 1)
    chol_leaf_kernel(const float* __restrict__ A, long long n, long long d, int jb, float* __restrict__ U,
                     float* __restrict__ U_hi, float* __restrict__ U_lo, float* __restrict__ UT_hi,
                     float* __restrict__ UT_lo) {
    extern __shared__ __align__(16) uint8_t leaf_raw[];
    LeafSmem& S = *reinterpret_cast<LeafSmem*>(leaf_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr unsigned FULL = 0xffffffffu;

    for (int e = tid; e < NB * NB; e += blockDim.x) {
        const int r = e >> 7, c = e & 127;
        S.a[r][c] = A[(long long)(jb + r) * n + jb + c];
        S.u[r][c] = 0.f;
    }
    __syncthreads();

    for (int kb = 3; kb >= 0; --kb) {
        const int rb = kb * 32;
        if (warp == 0) {
            // (a) UL-Cholesky of the 32x32 diagonal block, lane = row
            float dv[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) dv[c] = (c >= lane) ? S.a[rb + lane][rb + c] : 0.f;
#pragma unroll
            for (int k = 31; k >= 0; --k) {
                const float piv = __shfl_sync(FULL, dv[k], k);
                if (lane == 0 && !(piv > 0.f && isfinite(piv)))
                    record_status(isfinite(piv) ? GPTQ_ERR_NOT_PD : GPTQ_ERR_NONFINITE, jb + rb + k);
                const float sq = sqrtf(piv);
                const float rk = (lane < k) ? dv[k] / sq : ((lane == k) ? sq : 0.f);
                dv[k] = rk;
#pragma unroll
                for (int c = 0; c < k; ++c) dv[c] -= rk * __shfl_sync(FULL, rk, c);
            }
#pragma unroll
            for (int c = 0; c < 32; ++c)
                if (c >= lane) S.a[rb + lane][rb + c] = dv[c];
            __syncwarp();
            // (b) X = R^-1 of the 32x32 block, lane = column, back substitution from the bottom
            float xv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) xv[i] = 0.f;
#pragma unroll
            for (int i = 31; i >= 0; --i) {
                float s = 0.f;
#pragma unroll
                for (int m = i + 1; m < 32; ++m) s = fmaf(S.a[rb + i][rb + m], xv[m], s);
                const float rii = S.a[rb + i][rb + i];
                xv[i] = (i == lane) ? 1.f / rii : ((i < lane) ? -s / rii : 0.f);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) S.xinv[kb][i][lane] = xv[i];
        }
        __syncthreads();
        if (kb == 0) break;
        // (c) panel: R[0:rb, rb:rb+32] = A[0:rb, rb:rb+32] X^T
        float pv[6];
#pragma unroll
        for (int it = 0; it < 6; ++it) {
            const int e = tid + it * 512;
            pv[it] = 0.f;
            if (e < rb * 32) {
                const int r = e >> 5, c = e & 31;
                float s = 0.f;
#pragma unroll
                for (int k = 0; k < 32; ++k) s = fmaf(S.a[r][rb + k], S.xinv[kb][c][k], s);
                pv[it] = s;
            }
        }
        __syncthreads();
#pragma unroll
        for (int it = 0; it < 6; ++it) {
            const int e = tid + it * 512;
            if (e < rb * 32) S.a[e >> 5][rb + (e & 31)] = pv[it];
        }
        __syncthreads();
        // (d) A[0:rb, 0:rb] -= P P^T on the upper triangle
        for (int e = tid; e < rb * rb; e += blockDim.x) {
            const int r = e / rb, c = e % rb;
            if (r > c) continue;
            float s = 0.f;
#pragma unroll
            for (int k = 0; k < 32; ++k) s = fmaf(S.a[r][rb + k], S.a[c][rb + k], s);
            S.a[r][c] -= s;
        }
        __syncthreads();
    }

    // inverse of the 128x128 R from the four 32-block inverses
    for (int e = tid; e < 4 * 1024; e += blockDim.x) {
        const int kb = e >> 10, i = (e >> 5) & 31, j = e & 31;
        S.u[kb * 32 + i][kb * 32 + j] = S.xinv[kb][i][j];
    }
    __syncthreads();
    for (int ib = 2; ib >= 0; --ib) {
        const int nj = 3 - ib;  // block columns ib+1 .. 3
        for (int e = tid; e < nj * 1024; e += blockDim.x) {
            const int jj = e >> 10, r = (e >> 5) & 31, c = e & 31;
            const int jb2 = ib + 1 + jj;
            float s = 0.f;
            for (int kb2 = ib + 1; kb2 <= jb2; ++kb2) {
#pragma unroll 8
                for (int m = 0; m < 32; ++m)
                    s = fmaf(S.a[ib * 32 + r][kb2 * 32 + m], S.u[kb2 * 32 + m][jb2 * 32 + c], s);
            }
            S.tmp[jj][r][c] = s;
        }
        __syncthreads();
        for (int e = tid; e < nj * 1024; e += blockDim.x) {
            const int jj = e >> 10, r = (e >> 5) & 31, c = e & 31;
            float s = 0.f;
#pragma unroll 8
            for (int m = 0; m < 32; ++m) s = fmaf(S.xinv[ib][r][m], S.tmp[jj][m][c], s);
            S.u[ib * 32 + r][(ib + 1 + jj) * 32 + c] = -s;
        }
        __syncthreads();
    }

    // outputs: row-major passes, then a transposed pass with consecutive threads on rows
    for (int e = tid; e < NB * NB; e += blockDim.x) {
        const int r = e >> 7, c = e & 127;
        const float v = S.u[r][c];
        const long long gr = jb + r, gc = jb + c;
        float h, l;
        split_tf32(v, h, l);
        U_hi[gr * n + gc] = h;
        U_lo[gr * n + gc] = l;
        if (gr < d && gc < d) U[gr * d + gc] = v;
    }
    for (int e = tid; e < NB * NB; e += blockDim.x) {
        const int c = e >> 7, r = e & 127;
        const float v = S.u[r][c];
        float h, l;
        split_tf32(v, h, l);
        UT_hi[(long long)(jb + c) * n + jb + r] = h;
        UT_lo[(long long)(jb + c) * n + jb + r] = l;
    }
}

}  // namespace gq

namespace gqh {

inline long long chol_n(long long d) { return (d + gq::NB - 1) / gq::NB * gq::NB; }

struct HinvWs {
    float *A, *RS_hi, *RS_lo, *U_hi, *U_lo, *UT_hi, *UT_lo, *TT_hi, *TT_lo, *AP_hi, *AP_lo, *scal;
};

inline size_t hinv_ws_bytes(long long d) {
    const long long n = chol_n(d);
    return (size_t)(9 * n * n + 2 * n * gq::NB + 64) * sizeof(float);
}

inline HinvWs hinv_ws_carve(void* ws, long long d) {
    const long long n = chol_n(d);
    float* p = static_cast<float*>(ws);
    HinvWs w;
    w.A = p;
    p += n * n;
    w.RS_hi = p;
    p += n * n;
    w.RS_lo = p;
    p += n * n;
    w.U_hi = p;
    p += n * n;
    w.U_lo = p;
    p += n * n;
    w.UT_hi = p;
    p += n * n;
    w.UT_lo = p;
    p += n * n;
    w.TT_hi = p;
    p += n * n;
    w.TT_lo = p;
    p += n * n;
    w.AP_hi = p;
    p += n * gq::NB;
    w.AP_lo = p;
    p += n * gq::NB;
    w.scal = p;
    return w;
}


// Enqueue the whole factorization.  Leaves U (public, d x d) and the splits of U
// (U_hi/U_lo row-major, UT_hi/UT_lo transposed; n x n) in the workspace.
inline cudaError_t hinv_run(const float* H, long long d, float damp_rel, float* U, void* ws,
                            cudaStream_t st) {
    const long long n = chol_n(d);
    const int T = (int)(n / gq::NB);
    HinvWs w = hinv_ws_carve(ws, d);
    {
        gqh::TimedScope ts__("diag_mean", st);
        gq::diag_mean_kernel<<<1, 1024, 0, st>>>(H, d, damp_rel, w.scal);
    }
    GQ_TRY(cudaGetLastError());
    {
        dim3 tb(32, 8), grid((unsigned)(n / 32), (unsigned)(n / 32));
        {
            gqh::TimedScope ts__("damp_copy", st);
            gq::damp_copy_kernel<<<grid, tb, 0, st>>>(H, d, n, w.scal, w.A);
        }
        GQ_TRY(cudaGetLastError());
    }
    const int leaf_smem = (int)sizeof(gq::LeafSmem);
    GQ_TRY(cudaFuncSetAttribute(gq::chol_leaf_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, leaf_smem));
    const uint64_t N = (uint64_t)n;
    for (int j = T - 1; j >= 0; --j) {
        const int jb = j * gq::NB;
        {
            gqh::TimedScope ts__("chol_leaf", st);
            gq::chol_leaf_kernel<<<1, 512, leaf_smem, st>>>(w.A, n, d, jb, U, w.U_hi, w.U_lo, w.UT_hi, w.UT_lo);
        }
        GQ_TRY(cudaGetLastError());
        if (j == 0) break;
        {
            gqh::TimedScope ts__("split_panel", st);
            gq::split_panel_kernel<<<(unsigned)std::min<long long>((jb * 128LL + 255) / 256, 4096), 256, 0, st>>>(
                w.A, n, jb, jb, w.AP_hi, w.AP_lo);
        }
        GQ_TRY(cudaGetLastError());
        {   // panel: RS[0:jb, jb:jb+128] = AP * X^T, X = U block (row-major split)
            gq::GemmArgs p = gemm_args(jb, gq::NB, gq::NB);
            p.b_row0 = jb;
            p.b_col0 = jb;
            p.S_hi = w.RS_hi;
            p.S_lo = w.RS_lo;
            p.lds = n;
            p.s_col0 = jb;
            Mat ah{w.AP_hi, (uint64_t)jb, 128, 128}, al{w.AP_lo, (uint64_t)jb, 128, 128};
            Mat bh{w.U_hi, N, N, N}, bl{w.U_lo, N, N, N};
            GQ_TRY((launch_gemm<gq::KIND_TF32X3, 128, 3>(ah, al, bh, bl, p, 1, st, "chol_panel")));
        }
        {   // update: A[0:jb, 0:jb] -= RS_panel RS_panel^T (upper tiles)
            gq::GemmArgs p = gemm_args(jb, jb, gq::NB);
            p.a_col0 = jb;
            p.b_col0 = jb;
            p.triangular = 1;
            p.alpha = -1.f;
            p.beta = 1.f;
            p.C = w.A;
            p.ldc = n;
            p.write_c = 1;
            Mat rh{w.RS_hi, N, N, N}, rl{w.RS_lo, N, N, N};
            GQ_TRY((launch_gemm<gq::KIND_TF32X3, 128, 3>(rh, rl, rh, rl, p, 1, st, "chol_update")));
        }
    }
    // U = R^-1 by doubling
    Mat rsh{w.RS_hi, N, N, N}, rsl{w.RS_lo, N, N, N};
    Mat uth{w.UT_hi, N, N, N}, utl{w.UT_lo, N, N, N};
    Mat uh{w.U_hi, N, N, N}, ul{w.U_lo, N, N, N};
    Mat tth{w.TT_hi, N, N, N}, ttl{w.TT_lo, N, N, N};
    for (long long s = gq::NB; s < n; s *= 2) {
        const long long full = n / (2 * s);
        const long long rem = n - full * 2 * s;
        for (int part = 0; part < 2; ++part) {
            long long r0, cs, batch;
            if (part == 0) {
                r0 = 0;
                cs = s;
                batch = full;
            } else {
                if (rem <= s) break;
                r0 = full * 2 * s;
                cs = rem - s;
                batch = 1;
            }
            if (batch <= 0) continue;
            const int zs = (int)(2 * s);
            {   // T = B U_c, stored transposed in TT at (r0+s+j, r0+i)
                gq::GemmArgs p = gemm_args((int)s, (int)cs, (int)cs);
                p.a_row0 = (int)r0;
                p.a_col0 = (int)(r0 + s);
                p.a_zrow = p.a_zcol = zs;
                p.b_row0 = (int)(r0 + s);
                p.b_col0 = (int)(r0 + s);
                p.b_zrow = p.b_zcol = zs;
                p.k_to_n1 = 1;
                p.T_hi = w.TT_hi;
                p.T_lo = w.TT_lo;
                p.ldt = n;
                p.t_row0 = (int)(r0 + s);
                p.t_col0 = (int)r0;
                p.t_zrow = p.t_zcol = zs;
                GQ_TRY((launch_gemm<gq::KIND_TF32X3, 128, 3>(rsh, rsl, uth, utl, p, (int)batch, st, "inv_bu")));
            }
            {   // U_b = -U_a T -> U (public, clipped), U split, UT split
                gq::GemmArgs p = gemm_args((int)s, (int)cs, (int)s);
                p.a_row0 = (int)r0;
                p.a_col0 = (int)r0;
                p.a_zrow = p.a_zcol = zs;
                p.b_row0 = (int)(r0 + s);
                p.b_col0 = (int)r0;
                p.b_zrow = p.b_zcol = zs;
                p.k_from_m0 = 1;
                p.alpha = -1.f;
                p.C = U;
                p.ldc = d;
                p.c_row0 = (int)r0;
                p.c_col0 = (int)(r0 + s);
                p.c_zrow = p.c_zcol = zs;
                p.c_lim_rows = (int)d;
                p.c_lim_cols = (int)d;
                p.write_c = 1;
                p.S_hi = w.U_hi;
                p.S_lo = w.U_lo;
                p.lds = n;
                p.s_row0 = (int)r0;
                p.s_col0 = (int)(r0 + s);
                p.s_zrow = p.s_zcol = zs;
                p.T_hi = w.UT_hi;
                p.T_lo = w.UT_lo;
                p.ldt = n;
                p.t_row0 = (int)(r0 + s);
                p.t_col0 = (int)r0;
                p.t_zrow = p.t_zcol = zs;
                GQ_TRY((launch_gemm<gq::KIND_TF32X3, 128, 3>(uh, ul, tth, ttl, p, (int)batch, st, "inv_ub")));
            }
        }
    }
    {
        const long long tot = d * d;
        {
            gqh::TimedScope ts__("zero_lower", st);
            gq::zero_lower_blocks_kernel<<<(unsigned)std::min<long long>((tot + 255) / 256, 8192), 256, 0, st>>>(U, d);
        }
        GQ_TRY(cudaGetLastError());
    }
    return cudaSuccess;
}

}  // namespace gqh
