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
// Works on the index-reversed block P = J A_jj J, for which the UL factor becomes an
// ordinary lower Cholesky factor: A_jj = R R^T with R = J L J, and X_jj = R^-1 = J L^-1 J.
// Blocked by 32.  For each diagonal 32-block one warp runs Gaussian elimination on
// [P_kk | I] with unscaled pivot rows (lane = row): afterwards L_kk = L_u D^1/2 and
// L_kk^-1 = D^-1/2 E, where E is the accumulated row-operation matrix.  All warps then
// form the panel L_rk = P_rk L_kk^-T and the rank-32 update of the trailing lower
// triangle, on 4x4 register micro-tiles fed from transposed copies of L and of the
// diagonal inverses.  The inverse is assembled along block diagonals:
// X_ij = -X_ii sum_{k=j}^{i-1} L_ik X_kj.
// Writes X_jj (upper, zeros below the diagonal) to the public U (clipped to d), its
// row-major tf32 split (U_hi/U_lo) and its transposed split (UT_hi/UT_lo).
constexpr int LS = NB + 4;   // leaf smem row stride (16-byte aligned rows)

struct LeafSmem {
    float P[NB][LS];         // reversed block; lower triangle holds L after the factorization
    float X[NB][LS];         // L^-1 (lower); upper blocks hold temporaries
    float LT[NB][LS];        // L transposed: LT[m][r] = L[r][m]
    float XDT[4][32][36];    // diagonal inverses transposed: XDT[kb][m][j] = X_kk[j][m]
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__global__ void __launch_bounds__(512, 1)
    chol_leaf_kernel(const float* __restrict__ A, long long n, long long d, int jb, float* __restrict__ U,
                     float* __restrict__ U_hi, float* __restrict__ U_lo, float* __restrict__ UT_hi,
                     float* __restrict__ UT_lo) {
    extern __shared__ __align__(16) uint8_t leaf_raw[];
    LeafSmem& S = *reinterpret_cast<LeafSmem*>(leaf_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr unsigned FULL = 0xffffffffu;

    // P[127-r][127-c] = A[r][c]: coalesced reads of the whole diagonal tile (both
    // triangles were updated); only P's lower triangle (A's upper) is used.
    for (int e = tid; e < NB * NB; e += blockDim.x) {
        const int r = e >> 7, c = e & 127;
        S.P[127 - r][127 - c] = A[(long long)(jb + r) * n + jb + c];
        S.X[r][c] = 0.f;
    }
    __syncthreads();

    for (int kb = 0; kb < 4; ++kb) {
        const int k0 = kb * 32;
        if (warp == 0) {
            // (a) elimination of [P_kk | I] with unscaled pivot rows; lane = row
            float pr[32], xr[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                pr[j] = (j <= lane) ? S.P[k0 + lane][k0 + j] : S.P[k0 + j][k0 + lane];
                xr[j] = (j == lane) ? 1.f : 0.f;
            }
            float my_rinv = 0.f;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                // pivot row k (unscaled) is broadcast element by element with shuffles
                const float piv = __shfl_sync(FULL, pr[k], k);
                if (lane == 0 && !(piv > 0.f && isfinite(piv)))
                    record_status(isfinite(piv) ? GPTQ_ERR_NOT_PD : GPTQ_ERR_NONFINITE, jb + 127 - (k0 + k));
                const float rinv = rsqrtf(piv);
                const bool below = lane > k;
                const float f = below ? pr[k] * rinv * rinv : 0.f;   // P_ik / P_kk
                my_rinv = (lane == k) ? rinv : my_rinv;
#pragma unroll
                for (int j = k + 1; j < 32; ++j) pr[j] = fmaf(-f, __shfl_sync(FULL, pr[j], k), pr[j]);
#pragma unroll
                for (int j = 0; j <= k; ++j) xr[j] = fmaf(-f, __shfl_sync(FULL, xr[j], k), xr[j]);
                if (below) pr[k] *= rinv;   // L[lane][k] = P_ik / sqrt(P_kk)
            }
            // lane i: L[i][j] = pr[j] (j < i), L[i][i] = pivot * rinv, row i of L^-1 = rinv * xr
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                if (j <= lane) {
                    const float lij = (j == lane) ? pr[j] * my_rinv : pr[j];
                    const float xij = xr[j] * my_rinv;
                    S.P[k0 + lane][k0 + j] = lij;
                    S.LT[k0 + j][k0 + lane] = lij;
                    S.X[k0 + lane][k0 + j] = xij;
                    S.XDT[kb][j][lane] = xij;
                } else {
                    S.XDT[kb][j][lane] = 0.f;
                }
            }
        }
        __syncthreads();
        if (kb == 3) break;
        const int t0 = k0 + 32;
        const int rows = NB - t0;
        // (b) panel: L[r][k0+j] = sum_m P[r][k0+m] X_kk[j][m]; task = (row, 4 columns)
        for (int base = 0; base < rows * 8; base += 512) {
            const int task = base + tid;
            const int r = t0 + (task >> 3), j4 = (task & 7) * 4;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (task < rows * 8) {
#pragma unroll 8
                for (int m = 0; m < 32; ++m) {
                    const float pv = S.P[r][k0 + m];
                    const float4 xv = ld4(&S.XDT[kb][m][j4]);
                    acc.x = fmaf(pv, xv.x, acc.x);
                    acc.y = fmaf(pv, xv.y, acc.y);
                    acc.z = fmaf(pv, xv.z, acc.z);
                    acc.w = fmaf(pv, xv.w, acc.w);
                }
            }
            __syncwarp();
            if (task < rows * 8) {
                *reinterpret_cast<float4*>(&S.P[r][k0 + j4]) = acc;
                S.LT[k0 + j4 + 0][r] = acc.x;
                S.LT[k0 + j4 + 1][r] = acc.y;
                S.LT[k0 + j4 + 2][r] = acc.z;
                S.LT[k0 + j4 + 3][r] = acc.w;
            }
        }
        __syncthreads();
        // (c) trailing update of the lower triangle on 4x4 micro-tiles
        {
            const int T = rows >> 2;
            for (int task = tid; task < T * T; task += blockDim.x) {
                const int tr = task / T, tc = task % T;
                if (tc > tr) continue;
                const int r0 = t0 + 4 * tr, c0 = t0 + 4 * tc;
                float acc[4][4] = {};
#pragma unroll 4
                for (int m = 0; m < 32; ++m) {
                    const float4 a = ld4(&S.LT[k0 + m][r0]);
                    const float4 b = ld4(&S.LT[k0 + m][c0]);
                    const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float4 pv = ld4(&S.P[r0 + i][c0]);
                    pv.x -= acc[i][0];
                    pv.y -= acc[i][1];
                    pv.z -= acc[i][2];
                    pv.w -= acc[i][3];
                    *reinterpret_cast<float4*>(&S.P[r0 + i][c0]) = pv;
                }
            }
        }
        __syncthreads();
    }

    // inverse blocks below the diagonal, by block diagonals dd = i - j, 4x4 micro-tiles
    for (int dd = 1; dd < 4; ++dd) {
        const int nblk = 4 - dd;
        for (int task = tid; task < nblk * 64; task += blockDim.x) {
            // T_ij = sum_{m'=32j}^{32i-1} L[32i+r][m'] X[m'][32j+c] -> stored in X[32j+r][32i+c]
            const int jbk = task >> 6, ib = jbk + dd, tr = (task >> 3) & 7, tc = task & 7;
            const int r0 = 4 * tr, c0 = 4 * tc;
            float acc[4][4] = {};
            for (int m = 32 * jbk; m < 32 * ib; ++m) {
                const float4 a = ld4(&S.LT[m][32 * ib + r0]);
                const float4 b = ld4(&S.X[m][32 * jbk + c0]);
                const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<float4*>(&S.X[32 * jbk + r0 + i][32 * ib + c0]) =
                    make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        }
        __syncthreads();
        for (int task = tid; task < nblk * 64; task += blockDim.x) {
            // X_ij[r][c] = -sum_m X_ii[r][m] T[m][c]
            const int jbk = task >> 6, ib = jbk + dd, tr = (task >> 3) & 7, tc = task & 7;
            const int r0 = 4 * tr, c0 = 4 * tc;
            float acc[4][4] = {};
#pragma unroll 4
            for (int m = 0; m < 32; ++m) {
                const float4 a = ld4(&S.XDT[ib][m][r0]);
                const float4 b = ld4(&S.X[32 * jbk + m][32 * ib + c0]);
                const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<float4*>(&S.X[32 * ib + r0 + i][32 * jbk + c0]) =
                    make_float4(-acc[i][0], -acc[i][1], -acc[i][2], -acc[i][3]);
        }
        __syncthreads();
    }

    // U block = J X J (upper): U[r][c] = X[127-r][127-c] for r <= c; 4 columns per thread
    for (int task = tid; task < NB * 32; task += blockDim.x) {
        const int r = task >> 5, c = (task & 31) * 4;
        const float4 xv = ld4(&S.X[127 - r][124 - c]);   // columns 124-c .. 127-c, reversed below
        float v[4] = {xv.w, xv.z, xv.y, xv.x};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (r > c + i) v[i] = 0.f;
        float h[4], l[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) split_tf32(v[i], h[i], l[i]);
        const long long gr = jb + r, gc = jb + c;
        *reinterpret_cast<float4*>(U_hi + gr * n + gc) = make_float4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<float4*>(U_lo + gr * n + gc) = make_float4(l[0], l[1], l[2], l[3]);
        if (gr < d) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (gc + i < d) U[gr * d + gc + i] = v[i];
        }
    }
    // UT[c][r..r+3] = U[r..r+3][c] = X[127-r-i][127-c]; consecutive lanes take consecutive c
    // so the shared-memory reads run along rows of X (conflict-free)
    for (int task = tid; task < NB * 32; task += blockDim.x) {
        const int r = (task >> 7) * 4, c = task & 127;
        float v[4], h[4], l[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = (r + i <= c) ? S.X[127 - r - i][127 - c] : 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) split_tf32(v[i], h[i], l[i]);
        const long long off = (long long)(jb + c) * n + jb + r;
        *reinterpret_cast<float4*>(UT_hi + off) = make_float4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<float4*>(UT_lo + off) = make_float4(l[0], l[1], l[2], l[3]);
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
    GQ_TRY(ensure_smem_attr(reinterpret_cast<const void*>(gq::chol_leaf_kernel), leaf_smem));
    const uint64_t N = (uint64_t)n;
    for (int j = T - 1; j >= 0; --j) {
        const int jb = j * gq::NB;
        {
            gqh::TimedScope ts__("chol_leaf", st);
            gq::chol_leaf_kernel<<<1, 512, leaf_smem, st>>>(w.A, n, d, jb, U, w.U_hi, w.U_lo, w.UT_hi, w.UT_lo);
        }
        GQ_TRY(cudaGetLastError());
        if (j == 0) break;
        if (j == T - 1) {   // later panels are split by the previous update's epilogue
            gqh::TimedScope ts__("split_panel", st);
            gq::split_panel_kernel<<<(unsigned)std::min<long long>((jb * 128LL + 255) / 256, 4096), 256, 0, st>>>(
                w.A, n, jb, jb, w.AP_hi, w.AP_lo);
        }
        GQ_TRY(cudaGetLastError());
        {   // panel: RS[0:jb, jb:jb+128] = AP * X^T, X = U block (row-major split)
            gq::GemmArgs p = gemm_args(jb, gq::NB, gq::NB);
            p.b_row0 = jb;
            p.b_col0 = jb;
            p.s_col0 = jb;
            EpiMats o;
            o.s_hi = Mat{w.RS_hi, N, N, N};
            o.s_lo = Mat{w.RS_lo, N, N, N};
            Mat ah{w.AP_hi, (uint64_t)jb, 128, 128}, al{w.AP_lo, (uint64_t)jb, 128, 128};
            Mat bh{w.U_hi, N, N, N}, bl{w.U_lo, N, N, N};
            GQ_TRY((launch_gemm<gq::KIND_TF32X3, 2>(ah, al, bh, bl, o, p, 1, st, "chol_panel")));
        }
        {   // update: A[0:jb, 0:jb] -= RS_panel RS_panel^T (upper tiles)
            gq::GemmArgs p = gemm_args(jb, jb, gq::NB);
            p.a_col0 = jb;
            p.b_col0 = jb;
            p.triangular = 1;
            p.alpha = -1.f;
            p.beta = 1.f;
            p.write_c = 1;
            EpiMats o;
            o.c = Mat{w.A, N, N, N};
            if (j >= 2) {   // tiles of block column j-1 above its diagonal also write the next panel's split
                p.s_tile_n = j - 1;
                p.s_col0 = -(j - 1) * gq::NB;
                o.s_hi = Mat{w.AP_hi, (uint64_t)(jb - gq::NB), 128, 128};
                o.s_lo = Mat{w.AP_lo, (uint64_t)(jb - gq::NB), 128, 128};
            }
            Mat rh{w.RS_hi, N, N, N}, rl{w.RS_lo, N, N, N};
            GQ_TRY((launch_gemm<gq::KIND_TF32X3, 2>(rh, rl, rh, rl, o, p, 1, st, "chol_update")));
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
                p.t_row0 = (int)(r0 + s);
                p.t_col0 = (int)r0;
                p.t_zrow = p.t_zcol = zs;
                EpiMats o;
                o.t_hi = Mat{w.TT_hi, N, N, N};
                o.t_lo = Mat{w.TT_lo, N, N, N};
                GQ_TRY((launch_gemm<gq::KIND_TF32X3, 2>(rsh, rsl, uth, utl, o, p, (int)batch, st, "inv_bu")));
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
                p.c_row0 = (int)r0;
                p.c_col0 = (int)(r0 + s);
                p.c_zrow = p.c_zcol = zs;
                p.write_c = 1;
                p.s_row0 = (int)r0;
                p.s_col0 = (int)(r0 + s);
                p.s_zrow = p.s_zcol = zs;
                p.t_row0 = (int)(r0 + s);
                p.t_col0 = (int)r0;
                p.t_zrow = p.t_zcol = zs;
                EpiMats o;
                o.c = Mat{U, (uint64_t)d, (uint64_t)d, (uint64_t)d};   // public U, clipped to d x d
                o.s_hi = Mat{w.U_hi, N, N, N};
                o.s_lo = Mat{w.U_lo, N, N, N};
                o.t_hi = Mat{w.UT_hi, N, N, N};
                o.t_lo = Mat{w.UT_lo, N, N, N};
                GQ_TRY((launch_gemm<gq::KIND_TF32X3, 2>(uh, ul, tth, ttl, o, p, (int)batch, st, "inv_ub")));
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
