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
//   scheduled on three streams: the chain carries leaf(j) and, for the next leaf, only the
//   128x128 products R_{j-1,j} and A_{j-1,j-1} -= R_{j-1,j} R_{j-1,j}^T; a high-priority
//   stream the rest of the panel and block columns j-1 and j-2; a low-priority stream the
//   Schur update of the block columns left of them (look-ahead of depth two).
//   and U = R^-1 by doubling on a fourth stream, each product as soon as its inputs exist:
//   for each diagonal pair [[R_a, B], [0, R_c]] of 128, 256, ... columns with known
//   inverses U_a, U_c:  U_b = -U_a (B U_c).
#pragma once
#include "gemm_tc.cuh"
#include "actorder.cuh"

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
// A = H + lambda I on the upper 128-block triangle (bi <= bj, one CTA per block), from
// H's upper triangle; diagonal blocks are symmetrised in full; indices >= d pad A with the
// identity.  The strictly lower blocks of A are never read by the factorization and are
// not written.
__global__ void __launch_bounds__(256) damp_copy_kernel(const float* __restrict__ H, long long d, long long n,
                                                        const float* __restrict__ lam, float* __restrict__ A) {
    const int bi = blockIdx.y, bj = blockIdx.x;
    if (bi > bj) return;
    const long long r0 = (long long)bi * NB, c0 = (long long)bj * NB;
    const float l = lam[0];
    if (bi < bj) {
        for (int e = threadIdx.x; e < NB * NB / 4; e += blockDim.x) {
            const int r = e >> 5, c = (e & 31) * 4;
            const long long i = r0 + r, j = c0 + c;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < d && j < d) {   // d % 4 == 0: a float4 is wholly inside or outside
                v = *reinterpret_cast<const float4*>(H + i * d + j);
                if (!(isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w)))
                    record_status(GPTQ_ERR_NONFINITE, i * d + j);
            }
            *reinterpret_cast<float4*>(A + i * n + j) = v;
        }
        return;
    }
    // diagonal block: A[i][j] = H[min(i,j)][max(i,j)] (the few transposed reads are strided)
    for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
        const int r = e >> 7, c = e & 127;
        const long long i = r0 + r, j = c0 + c;
        float v = 0.f;
        if (i < d && j < d) {
            v = (r <= c) ? H[i * d + j] : H[j * d + i];
            if (r <= c && !isfinite(v)) record_status(GPTQ_ERR_NONFINITE, i * d + j);
        }
        if (i == j) v = (i < d) ? v + l : 1.f;
        A[i * n + j] = v;
    }
}

// The damped copy of damp_copy_kernel for the permuted Hessian: A[i][j] =
// H[perm[i]][perm[j]] (+ lambda on the diagonal) for j >= the start of i's 128-block,
// identity padding past d.  One CTA per row of A: it reads one row of H, so every
// sector of H is fetched once.  H must hold both triangles.
__global__ void __launch_bounds__(256) damp_copy_perm_kernel(const float* __restrict__ H,
                                                             const int* __restrict__ perm, long long d, long long n,
                                                             const float* __restrict__ lam, float* __restrict__ A) {
    const long long i = blockIdx.x;
    const long long j0 = (i / NB) * NB;
    float* out = A + i * n;
    if (i >= d) {
        for (long long j = j0 + threadIdx.x; j < n; j += blockDim.x) out[j] = (i == j) ? 1.f : 0.f;
        return;
    }
    const float l = lam[0];
    const float* src = H + (long long)checked_index(perm, i, d) * d;
    for (long long j = j0 + threadIdx.x; j < n; j += blockDim.x) {
        float v = 0.f;
        if (j < d) {
            v = src[checked_index(perm, j, d)];
            if (!isfinite(v)) record_status(GPTQ_ERR_NONFINITE, i * d + j);
            if (i == j) v += l;
        }
        out[j] = v;
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
// written in full by chol_diag_out_kernel).
__global__ void __launch_bounds__(256) zero_lower_blocks_kernel(float* __restrict__ U, long long d) {
    const int bi = blockIdx.y, bj = blockIdx.x;   // one CTA per 128-block, strictly lower only
    if (bi <= bj) return;
    const long long r0 = (long long)bi * NB, c0 = (long long)bj * NB;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e = threadIdx.x; e < NB * NB / 4; e += blockDim.x) {
        const long long i = r0 + (e >> 5), j = c0 + (e & 31) * 4;
        if (i < d && j < d) *reinterpret_cast<float4*>(U + i * d + j) = z;   // d % 4 == 0
    }
}

// Leaf: factor and invert one 128x128 diagonal block of A in shared memory.
// Works on the index-reversed block P = J A_jj J, for which the UL factor becomes an
// ordinary lower Cholesky factor: A_jj = R R^T with R = J L J, and X_jj = R^-1 = J L^-1 J.
//
// Right-looking, blocked by 32 columns.  For panel kb (columns k0 = 32 kb .. k0 + 31):
//   A. one warp factors the 32x32 diagonal block in registers, lane = row.  The only
//      dependency from one pivot to the next is one shuffle of the next pivot, which each
//      lane keeps up to date from its own multipliers (the broadcasts of the multipliers to
//      the other rows are off that chain); 1/L_kk = rsqrt with one Newton step.
//   B. the rows below the block (one thread per row, 32 - 96 rows) solve against L_kk by
//      substitution with the reciprocals of step A; meanwhile one otherwise idle warp forms
//      X_kk = L_kk^-1 by forward substitution (lane = column).
//   C. all threads apply the rank-32 update of the trailing lower triangle on 4x4
//      register micro-tiles.
// Then the off-diagonal blocks of X = L^-1, block row by block row:
// X_ij = -X_ii sum_{k=j}^{i-1} L_ik X_kj, the sums first (kept in X's free upper blocks).
// Writes X_jj (upper, zeros below the diagonal) as U_hi = tf32(X_jj) and U_lo = X_jj - U_hi
// (exact, not rounded: the tensor pipe reads only its tf32 part); U_hi + U_lo restores
// X_jj exactly for chol_diag_out_kernel.
constexpr int LS = NB + 4;   // leaf smem row stride (16-byte aligned rows)
constexpr int LEAF_THREADS = 512;
static_assert(NB * NB / 4 == 8 * LEAF_THREADS && NB * 32 == 8 * LEAF_THREADS, "leaf load and store loops");

struct LeafSmem {
    float P[NB][LS];         // reversed block; lower triangle holds the Schur complement
    float X[NB][LS];         // L^-1 (lower); blocks above the diagonal hold the block-row sums
    float LT[NB][LS];        // L transposed: LT[m][r] = L[r][m]
    float XDT[4][32][36];    // diagonal inverses transposed: XDT[i][m][r] = X_ii[r][m]
    float rinv[NB];          // 1 / L_kk
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// A. Factor the 32x32 diagonal block at (k0, k0) with one warp; lane i holds row k0 + i.
// Writes L_kk (lower, zeros above) to P and LT, and 1/L_kk to rinv.
__device__ __forceinline__ void leaf_diag_factor(LeafSmem& S, int k0, int lane, int jb) {
    constexpr unsigned FULL = 0xffffffffu;
    float a[32];
#pragma unroll
    for (int j4 = 0; j4 < 8; ++j4) {
        const float4 v = ld4(&S.P[k0 + lane][k0 + 4 * j4]);
        a[4 * j4 + 0] = v.x;
        a[4 * j4 + 1] = v.y;
        a[4 * j4 + 2] = v.z;
        a[4 * j4 + 3] = v.w;
    }
    // this lane's diagonal entry, kept current with the lane's own multipliers
    float dg = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) dg = (lane == j) ? a[j] : dg;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const float p = __shfl_sync(FULL, dg, k);   // pivot: P_kk after pivots 0..k-1
        if (lane == 0 && !(p > 0.f && isfinite(p)))
            record_status(isfinite(p) ? GPTQ_ERR_NOT_PD : GPTQ_ERR_NONFINITE, jb + 127 - (k0 + k));
        float r = rsqrtf(p);
        r = r * fmaf(-0.5f * p * r, r, 1.5f);       // one Newton step for 1/sqrt(p)
        const float l = (lane == k) ? p * r : a[k] * r;   // L_kk = sqrt(p); L_ik = P_ik / L_kk
        a[k] = l;
        if (lane > k) dg = fmaf(-l, l, dg);
        if (lane == k) S.rinv[k0 + k] = r;
#pragma unroll
        for (int j = k + 1; j < 32; ++j) {
            const float lj = __shfl_sync(FULL, l, j);
            a[j] = fmaf(-l, lj, a[j]);              // P_ij -= L_ik L_jk (meaningful for lanes >= j)
        }
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float v = (j <= lane) ? a[j] : 0.f;
        S.P[k0 + lane][k0 + j] = v;
        S.LT[k0 + j][k0 + lane] = v;
    }
}

// B. Rows k0+32 .. 127 (one thread each): L_i,kb = P_i,kb L_kk^-T by substitution.
__device__ __forceinline__ void leaf_panel_solve(LeafSmem& S, int k0, int i) {
    float a[32];
#pragma unroll
    for (int j4 = 0; j4 < 8; ++j4) {
        const float4 v = ld4(&S.P[i][k0 + 4 * j4]);
        a[4 * j4 + 0] = v.x;
        a[4 * j4 + 1] = v.y;
        a[4 * j4 + 2] = v.z;
        a[4 * j4 + 3] = v.w;
    }
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const float l = a[k] * S.rinv[k0 + k];
        a[k] = l;
#pragma unroll
        for (int j4 = (k + 1) >> 2; j4 < 8; ++j4) {
            const float4 c4 = ld4(&S.LT[k0 + k][k0 + 4 * j4]);   // L_jk for j = 4 j4 ..
            if (4 * j4 + 0 > k) a[4 * j4 + 0] = fmaf(-l, c4.x, a[4 * j4 + 0]);
            if (4 * j4 + 1 > k) a[4 * j4 + 1] = fmaf(-l, c4.y, a[4 * j4 + 1]);
            if (4 * j4 + 2 > k) a[4 * j4 + 2] = fmaf(-l, c4.z, a[4 * j4 + 2]);
            if (4 * j4 + 3 > k) a[4 * j4 + 3] = fmaf(-l, c4.w, a[4 * j4 + 3]);
        }
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) S.LT[k0 + j][i] = a[j];
}

// C. Rank-32 update of the trailing lower triangle (rows and columns >= k0 + 32) with the
// panel just factored; 4x4 micro-tiles on the lower triangle of tiles only.
__device__ __forceinline__ void leaf_trailing_update(LeafSmem& S, int k0, int tid) {
    const int t0 = k0 + 32, tn = (NB - t0) >> 2;
    const int ntask = tn * (tn + 1) / 2;
    for (int task = tid; task < ntask; task += LEAF_THREADS) {
        int tr = (int)((sqrtf(8.f * (float)task + 1.f) - 1.f) * 0.5f);
        while (tr * (tr + 1) / 2 > task) --tr;
        while ((tr + 1) * (tr + 2) / 2 <= task) ++tr;
        const int tc = task - tr * (tr + 1) / 2;
        const int r0 = t0 + 4 * tr, c0 = t0 + 4 * tc;
        float acc[4][4] = {};
#pragma unroll 8
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

// X_ii = L_ii^-1 by forward substitution, one warp, lane = column j:
// x_m = (delta_mj - sum_{m' < m} L_mm' x_m') / L_mm, with 1/L_mm from step A.
__device__ __forceinline__ void leaf_diag_inverse(LeafSmem& S, int i, int lane) {
    const int k0 = 32 * i;
    float x[32], s[32];
#pragma unroll
    for (int m = 0; m < 32; ++m) s[m] = 0.f;
#pragma unroll
    for (int m = 0; m < 32; ++m) {
        x[m] = (((m == lane) ? 1.f : 0.f) - s[m]) * S.rinv[k0 + m];
#pragma unroll
        for (int q4 = (m + 1) >> 2; q4 < 8; ++q4) {
            const float4 l4 = ld4(&S.LT[k0 + m][k0 + 4 * q4]);   // L_{q,m} for q = 4 q4 ..
            if (4 * q4 + 0 > m) s[4 * q4 + 0] = fmaf(l4.x, x[m], s[4 * q4 + 0]);
            if (4 * q4 + 1 > m) s[4 * q4 + 1] = fmaf(l4.y, x[m], s[4 * q4 + 1]);
            if (4 * q4 + 2 > m) s[4 * q4 + 2] = fmaf(l4.z, x[m], s[4 * q4 + 2]);
            if (4 * q4 + 3 > m) s[4 * q4 + 3] = fmaf(l4.w, x[m], s[4 * q4 + 3]);
        }
    }
#pragma unroll
    for (int m = 0; m < 32; ++m) S.X[k0 + m][k0 + lane] = x[m];
#pragma unroll
    for (int m4 = 0; m4 < 8; ++m4)
        *reinterpret_cast<float4*>(&S.XDT[i][lane][4 * m4]) =
            make_float4(x[4 * m4], x[4 * m4 + 1], x[4 * m4 + 2], x[4 * m4 + 3]);
}

// Block row i of X = L^-1 with all threads: T_ij = sum_{k=j}^{i-1} L_ik X_kj into X's free
// upper block (j, i), then X_ij = -X_ii T_ij.  Block rows < i must be complete.
__device__ __forceinline__ void leaf_x_block_row(LeafSmem& S, int i, int tid) {
    for (int task = tid; task < 64 * i; task += LEAF_THREADS) {
        const int j = task >> 6, r0 = 4 * ((task >> 3) & 7), c0 = 4 * (task & 7);
        float acc[4][4] = {};
        for (int k = j; k < i; ++k) {
#pragma unroll 8
            for (int m = 0; m < 32; ++m) {
                const float4 a = ld4(&S.LT[32 * k + m][32 * i + r0]);   // L_ik[r][m]
                const float4 b = ld4(&S.X[32 * k + m][32 * j + c0]);    // X_kj[m][c]
                const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
            *reinterpret_cast<float4*>(&S.X[32 * j + r0 + u][32 * i + c0]) =
                make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
    }
    __syncthreads();
    for (int task = tid; task < 64 * i; task += LEAF_THREADS) {
        const int j = task >> 6, r0 = 4 * ((task >> 3) & 7), c0 = 4 * (task & 7);
        float acc[4][4] = {};
#pragma unroll 8
        for (int m = 0; m < 32; ++m) {
            const float4 a = ld4(&S.XDT[i][m][r0]);                   // X_ii[r][m]
            const float4 b = ld4(&S.X[32 * j + m][32 * i + c0]);      // T_ij[m][c]
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
            *reinterpret_cast<float4*>(&S.X[32 * i + r0 + u][32 * j + c0]) =
                make_float4(-acc[u][0], -acc[u][1], -acc[u][2], -acc[u][3]);
    }
    __syncthreads();
}

__global__ void __launch_bounds__(LEAF_THREADS, 1)
    chol_leaf_kernel(const float* __restrict__ A, long long n, int jb, float* __restrict__ U_hi,
                     float* __restrict__ U_lo) {
    extern __shared__ __align__(16) uint8_t leaf_raw[];
    LeafSmem& S = *reinterpret_cast<LeafSmem*>(leaf_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_trigger();

    // P[127-r][127-c] = A[r][c]: the whole diagonal tile, in two halves whose loads are all
    // issued before their stores
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float4 v[4];
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int e = tid + (4 * half + it) * LEAF_THREADS, r = e >> 5, c = (e & 31) * 4;
            v[it] = *reinterpret_cast<const float4*>(A + (long long)(jb + r) * n + jb + c);
        }
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int e = tid + (4 * half + it) * LEAF_THREADS, r = e >> 5, c = (e & 31) * 4;
            S.P[127 - r][127 - c] = v[it].x;
            S.P[127 - r][126 - c] = v[it].y;
            S.P[127 - r][125 - c] = v[it].z;
            S.P[127 - r][124 - c] = v[it].w;
        }
    }
    __syncthreads();

    for (int kb = 0; kb < 4; ++kb) {
        const int k0 = 32 * kb;
        if (warp == 0) leaf_diag_factor(S, k0, lane, jb);
        __syncthreads();
        if (tid >= 32 && tid < 32 + (NB - k0 - 32)) leaf_panel_solve(S, k0, k0 + tid);   // rows k0+32 ..
        else if (warp == 15) leaf_diag_inverse(S, kb, lane);
        __syncthreads();
        if (kb < 3) {
            leaf_trailing_update(S, k0, tid);
            __syncthreads();
        }
    }
    for (int i = 1; i < 4; ++i) leaf_x_block_row(S, i, tid);

    // U block = J X J (upper): U[r][c] = X[127-r][127-c] for r <= c; 4 columns per thread
#pragma unroll 2
    for (int it = 0; it < NB * 32 / LEAF_THREADS; ++it) {
        const int task = tid + it * LEAF_THREADS, r = task >> 5, c = (task & 31) * 4;
        const float4 xv = ld4(&S.X[127 - r][124 - c]);   // columns 124-c .. 127-c, reversed below
        float v[4] = {xv.w, xv.z, xv.y, xv.x};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (r > c + i) v[i] = 0.f;
        float h[4], l[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            h[i] = to_tf32(v[i]);
            l[i] = v[i] - h[i];
        }
        const long long off = (long long)(jb + r) * n + jb + c;
        *reinterpret_cast<float4*>(U_hi + off) = make_float4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<float4*>(U_lo + off) = make_float4(l[0], l[1], l[2], l[3]);
    }
}

// One CTA per diagonal block jb = 128 * (blk0 + blockIdx.x): X_jj = U_hi + U_lo (exact, as the leaf
// wrote them).  Writes X_jj to the public U (clipped to d) and its transposed tf32 split to
// UT_hi/UT_lo.
__global__ void __launch_bounds__(512)
    chol_diag_out_kernel(const float* __restrict__ U_hi, const float* __restrict__ U_lo, float* __restrict__ UT_hi,
                         float* __restrict__ UT_lo, float* __restrict__ U, long long n, long long d, int blk0) {
    extern __shared__ __align__(16) uint8_t dout_raw[];
    float (*Vs)[NB + 1] = reinterpret_cast<float (*)[NB + 1]>(dout_raw);
    const long long jb = (long long)(blk0 + blockIdx.x) * NB;
    for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
        const int r = e >> 7, c = e & 127;
        const long long off = (jb + r) * n + jb + c;
        const float v = U_hi[off] + U_lo[off];
        Vs[r][c] = v;
        if (jb + r < d && jb + c < d) U[(jb + r) * d + jb + c] = v;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
        const int c = e >> 7, r = e & 127;   // UT[c][r] = U[r][c]
        float h, l;
        split_tf32(Vs[r][c], h, l);
        UT_hi[(jb + c) * n + jb + r] = h;
        UT_lo[(jb + c) * n + jb + r] = l;
    }
}

}  // namespace gq

namespace gqh {

inline long long chol_n(long long d) { return (d + gq::NB - 1) / gq::NB * gq::NB; }

struct HinvWs {
    float *A, *RS_hi, *RS_lo, *U_hi, *U_lo, *UT_hi, *UT_lo, *TT_hi, *TT_lo, *AP_hi, *AP_lo, *scal;
    int* rank;   // inverse of a caller's permutation (permuted factorization only)
};

inline size_t hinv_ws_bytes(long long d) {
    const long long n = chol_n(d);
    return (size_t)(9 * n * n + 4 * n * gq::NB + 64 + n) * sizeof(float);
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
    w.AP_hi = p;   // two panel splits (block columns of either parity), n x 128 each
    p += 2 * n * gq::NB;
    w.AP_lo = p;
    p += 2 * n * gq::NB;
    w.scal = p;
    p += 64;
    w.rank = reinterpret_cast<int*>(p);
    return w;
}


// Enqueue the whole factorization.  Leaves U (public, d x d) and the splits of U
// (U_hi/U_lo row-major, UT_hi/UT_lo transposed; n x n) in the workspace.
inline cudaError_t hinv_run(const float* H, long long d, float damp_rel, float* U, void* ws,
                            cudaStream_t st, const int* perm = nullptr) {
    const long long n = chol_n(d);
    const int T = (int)(n / gq::NB);
    HinvWs w = hinv_ws_carve(ws, d);
    {
        gqh::TimedScope ts__("diag_mean", st);
        gq::diag_mean_kernel<<<1, 1024, 0, st>>>(H, d, damp_rel, w.scal);
    }
    GQ_TRY(cudaGetLastError());
    if (perm) {   // factor P^T Hd P: validate the permutation, then a gathering damped copy
        GQ_TRY(cudaMemsetAsync(w.rank, 0xFF, (size_t)d * sizeof(int), st));
        {
            gqh::TimedScope ts__("perm_invert", st);
            gq::perm_invert_kernel<<<(unsigned)((d + 255) / 256), 256, 0, st>>>(perm, d, w.rank);
        }
        GQ_TRY(cudaGetLastError());
        {
            gqh::TimedScope ts__("damp_copy_perm", st);
            gq::damp_copy_perm_kernel<<<(unsigned)n, 256, 0, st>>>(H, perm, d, n, w.scal, w.A);
        }
        GQ_TRY(cudaGetLastError());
    } else {
        const dim3 grid((unsigned)(n / gq::NB), (unsigned)(n / gq::NB));
        {
            gqh::TimedScope ts__("damp_copy", st);
            gq::damp_copy_kernel<<<grid, 256, 0, st>>>(H, d, n, w.scal, w.A);
        }
        GQ_TRY(cudaGetLastError());
    }
    const int leaf_smem = (int)sizeof(gq::LeafSmem);
    GQ_TRY(ensure_smem_attr(reinterpret_cast<const void*>(gq::chol_leaf_kernel), leaf_smem));
    const uint64_t N = (uint64_t)n;
    // Streams.  The chain stream carries, per block column j, only what the next leaf needs:
    //   leaf(j) -> C1: R_{j-1,j} = A_{j-1,j} X_jj^T (one 128x128 block of the panel)
    //           -> C2: A_{j-1,j-1} -= R_{j-1,j} R_{j-1,j}^T        -> leaf(j-1).
    // The near stream: P, the rest of the panel (rows 0 .. j-2); N, block column j-1 above its
    // diagonal block (and the tf32 split of the next panel); U2, block column j-2 with its
    // diagonal block.  The far stream: R, the Schur update of block columns 0 .. j-3.
    // Every block is updated in step order: C1(j) reads the panel split N(j+1) wrote; C2(j)
    // follows U2(j+1) on block (j-1, j-1); U2(j) follows R(j+1) on block column j-2.
    FactStreams fs;
    if (!fact_streams(&fs)) return cudaErrorUnknown;
    cudaEvent_t ev_start = fs.ev[0], ev_leaf = fs.ev[1], ev_P = fs.ev[2], ev_C1 = fs.ev[3], ev_N = fs.ev[4],
                ev_U2 = fs.ev[5], ev_R = fs.ev[6], ev_near = fs.ev[7], ev_far = fs.ev[8], ev_chain = fs.ev[9],
                ev_inv = fs.ev[10];
    cudaStream_t sc = fs.chain, sn = fs.near, sf = fs.far, si = fs.inv;
    {
        gqh::TimedScope ts__("zero_lower", st);   // the public U's strictly lower blocks
        const unsigned nb = (unsigned)((d + gq::NB - 1) / gq::NB);
        gq::zero_lower_blocks_kernel<<<dim3(nb, nb), 256, 0, st>>>(U, d);
    }
    GQ_TRY(cudaGetLastError());
    GQ_TRY(cudaEventRecord(ev_start, st));
    GQ_TRY(cudaStreamWaitEvent(sc, ev_start, 0));
    GQ_TRY(cudaStreamWaitEvent(sn, ev_start, 0));
    GQ_TRY(cudaStreamWaitEvent(sf, ev_start, 0));
    GQ_TRY(cudaStreamWaitEvent(si, ev_start, 0));
    const int side = std::max(1, num_sms() - 8);   // helper grids leave SMs to the chain
    Mat rh{w.RS_hi, N, N, N}, rl{w.RS_lo, N, N, N};
    Mat xh{w.U_hi, N, N, N}, xl{w.U_lo, N, N, N};
    float* ap_hi[2] = {w.AP_hi, w.AP_hi + n * gq::NB};
    float* ap_lo[2] = {w.AP_lo, w.AP_lo + n * gq::NB};
    // C -= RS(rows a_row0 ..) RS(rows b_row0 ..)^T over the panel of block column j
    auto schur = [&](int jb, int M, int Ncols, int b_row0, int c_row0, int c_col0, bool tri, cudaStream_t s_,
                     const char* name, int max_ctas, const EpiMats* extra_s, bool after) -> cudaError_t {
        gq::GemmArgs p = gemm_args(M, Ncols, gq::NB);
        p.a_row0 = c_row0;
        p.a_col0 = jb;
        p.b_row0 = b_row0;
        p.b_col0 = jb;
        p.alpha = -1.f;
        p.beta = 1.f;
        p.write_c = 1;
        p.c_row0 = c_row0;
        p.c_col0 = c_col0;
        p.triangular = tri ? 1 : 0;
        EpiMats o;
        if (extra_s) o = *extra_s;
        o.c = Mat{w.A, N, N, N};
        if (tri) return launch_gemm<gq::KIND_TF32X3, 2, 128, 4>(rh, rl, rh, rl, o, p, 1, s_, name, max_ctas, after);
        return launch_gemm<gq::KIND_TF32X3, 4, 32, 2>(rh, rl, rh, rl, o, p, 1, s_, name, max_ctas, after);
    };
    // RS(rows r0 .. r0+M, block column j) = AP(rows r0 ..) X_jj^T
    auto panel = [&](int jb, int r0, int M, cudaStream_t s_, const char* name, int max_ctas, bool after) {
        const int par = (jb / gq::NB) & 1;
        gq::GemmArgs p = gemm_args(M, gq::NB, gq::NB);
        p.a_row0 = r0;
        p.b_row0 = jb;
        p.b_col0 = jb;
        p.s_row0 = r0;
        p.s_col0 = jb;
        EpiMats o;
        o.s_hi = Mat{w.RS_hi, N, N, N};
        o.s_lo = Mat{w.RS_lo, N, N, N};
        Mat ah{ap_hi[par], (uint64_t)jb, 128, 128}, al{ap_lo[par], (uint64_t)jb, 128, 128};
        return launch_gemm<gq::KIND_TF32X3, 4, 32, 2>(ah, al, xh, xl, o, p, 1, s_, name, max_ctas, after);
    };
    // U = R^-1 by doubling, each product issued on the inverse stream as soon as its inputs
    // exist: for the diagonal pair [[R_a, B], [0, R_c]] of level s (a-half rows r0 .. r0+s,
    // c-half r0+s .. r0+s+cs) with inverses U_a and U_c known, T = B U_c (stored transposed) as
    // soon as the c-half is inverted and the panels of its block columns are formed, and
    // U_b = -U_a T once the a-half is inverted.  Only the products of the pairs that contain
    // block 0 wait for the last leaf.
    Mat uth{w.UT_hi, N, N, N}, utl{w.UT_lo, N, N, N};
    Mat tth{w.TT_hi, N, N, N}, ttl{w.TT_lo, N, N, N};
    const int dout_smem = (int)(gq::NB * (gq::NB + 1) * sizeof(float));
    GQ_TRY(ensure_smem_attr(reinterpret_cast<const void*>(gq::chol_diag_out_kernel), dout_smem));
    auto inv_bu = [&](long long s_, long long r0, long long cs) -> cudaError_t {   // T = B U_c -> TT
        gq::GemmArgs p = gemm_args((int)s_, (int)cs, (int)cs);
        p.a_row0 = (int)r0;
        p.a_col0 = (int)(r0 + s_);
        p.b_row0 = (int)(r0 + s_);
        p.b_col0 = (int)(r0 + s_);
        p.k_to_n1 = 1;
        p.t_row0 = (int)(r0 + s_);
        p.t_col0 = (int)r0;
        EpiMats o;
        o.t_hi = Mat{w.TT_hi, N, N, N};
        o.t_lo = Mat{w.TT_lo, N, N, N};
        const bool narrow = 4 * (s_ / gq::NB) * ((cs + gq::NB - 1) / gq::NB) <= num_sms();
        if (narrow) return launch_gemm<gq::KIND_TF32X3, 4, 32, 2>(rh, rl, uth, utl, o, p, 1, si, "inv_bu", side, true);
        return launch_gemm<gq::KIND_TF32X3, 2, 128, 4>(rh, rl, uth, utl, o, p, 1, si, "inv_bu", side, true);
    };
    auto inv_ub = [&](long long s_, long long r0, long long cs) -> cudaError_t {   // U_b = -U_a T
        gq::GemmArgs p = gemm_args((int)s_, (int)cs, (int)s_);
        p.a_row0 = (int)r0;
        p.a_col0 = (int)r0;
        p.b_row0 = (int)(r0 + s_);
        p.b_col0 = (int)r0;
        p.k_from_m0 = 1;
        p.alpha = -1.f;
        p.c_row0 = (int)r0;
        p.c_col0 = (int)(r0 + s_);
        p.write_c = 1;
        p.s_row0 = (int)r0;
        p.s_col0 = (int)(r0 + s_);
        p.t_row0 = (int)(r0 + s_);
        p.t_col0 = (int)r0;
        EpiMats o;
        o.c = Mat{U, (uint64_t)d, (uint64_t)d, (uint64_t)d};   // public U, clipped to d x d
        o.s_hi = Mat{w.U_hi, N, N, N};
        o.s_lo = Mat{w.U_lo, N, N, N};
        o.t_hi = Mat{w.UT_hi, N, N, N};
        o.t_lo = Mat{w.UT_lo, N, N, N};
        const bool narrow = 4 * (s_ / gq::NB) * ((cs + gq::NB - 1) / gq::NB) <= num_sms();
        if (narrow) return launch_gemm<gq::KIND_TF32X3, 4, 32, 2>(xh, xl, tth, ttl, o, p, 1, si, "inv_ub", side, true);
        return launch_gemm<gq::KIND_TF32X3, 2, 128, 4>(xh, xl, tth, ttl, o, p, 1, si, "inv_ub", side, true);
    };
    // the inverse work that becomes possible once leaf(j) and the panels of block column j exist
    auto inverse_step = [&](int j) -> cudaError_t {
        const long long jb = (long long)j * gq::NB;
        GQ_TRY(cudaStreamWaitEvent(si, ev_leaf, 0));
        {
            gqh::TimedScope ts__("chol_diag_out", si);
            gq::chol_diag_out_kernel<<<1, 512, dout_smem, si>>>(w.U_hi, w.U_lo, w.UT_hi, w.UT_lo, U, n, d, j);
        }
        GQ_TRY(cudaGetLastError());
        for (long long s_ = gq::NB; s_ < n; s_ *= 2)   // pairs whose a-half starts at block j
            if (jb % (2 * s_) == 0 && jb + s_ < n) GQ_TRY(inv_ub(s_, jb, std::min(s_, n - jb - s_)));
        if (j > 0) {
            GQ_TRY(cudaStreamWaitEvent(si, ev_P, 0));
            GQ_TRY(cudaStreamWaitEvent(si, ev_C1, 0));
        }
        for (long long s_ = gq::NB; s_ < n; s_ *= 2)   // pairs whose c-half starts at block j
            if (jb >= s_ && (jb - s_) % (2 * s_) == 0) GQ_TRY(inv_bu(s_, jb - s_, std::min(s_, n - jb)));
        return cudaSuccess;
    };
    for (int j = T - 1; j >= 0; --j) {
        const int jb = j * gq::NB;
        const int jn = jb - gq::NB;    // first column of block column j-1
        const int jn2 = jn - gq::NB;   // first column of block column j-2
        {
            gqh::TimedScope ts__("chol_leaf", sc);
            if (j == T - 1)   // follows the wait for the damped copy on the caller's stream
                GQ_TRY(launch_plain(gq::chol_leaf_kernel, dim3(1), dim3(gq::LEAF_THREADS), (size_t)leaf_smem, sc,
                                    (const float*)w.A, n, jb, w.U_hi, w.U_lo));
            else
                GQ_TRY(launch_pdl(gq::chol_leaf_kernel, dim3(1), dim3(gq::LEAF_THREADS), (size_t)leaf_smem, sc,
                                  (const float*)w.A, n, jb, w.U_hi, w.U_lo));
        }
        if (j == 0) {
            GQ_TRY(cudaEventRecord(ev_leaf, sc));
            GQ_TRY(inverse_step(0));
            break;
        }
        if (j == T - 1) {   // the first panel's tf32 split; later ones come from N
            gqh::TimedScope ts__("split_panel", sc);
            gq::split_panel_kernel<<<(unsigned)std::min<long long>((jb * 128LL + 255) / 256, 4096), 256, 0, sc>>>(
                w.A, n, jb, jb, ap_hi[j & 1], ap_lo[j & 1]);
            GQ_TRY(cudaGetLastError());
        }
        GQ_TRY(cudaEventRecord(ev_leaf, sc));
        // near stream: the panel's rows 0 .. j-2
        GQ_TRY(cudaStreamWaitEvent(sn, ev_leaf, 0));
        if (jn > 0) GQ_TRY(panel(jb, 0, jn, sn, "chol_panel", side, true));
        GQ_TRY(cudaEventRecord(ev_P, sn));
        // chain: C1, C2
        GQ_TRY(cudaStreamWaitEvent(sc, ev_N, 0));
        GQ_TRY(panel(jb, jn, gq::NB, sc, "chol_chain_r", 0, true));
        GQ_TRY(cudaEventRecord(ev_C1, sc));
        GQ_TRY(cudaStreamWaitEvent(sc, ev_U2, 0));
        GQ_TRY(schur(jb, gq::NB, gq::NB, jn, jn, jn, false, sc, "chol_chain_d", 0, nullptr, true));
        if (jn > 0) {
            // near stream: N(j) = block column j-1 above its diagonal block + the next panel's split
            GQ_TRY(cudaStreamWaitEvent(sn, ev_C1, 0));
            EpiMats so;
            so.s_hi = Mat{ap_hi[(j - 1) & 1], (uint64_t)jn, 128, 128};
            so.s_lo = Mat{ap_lo[(j - 1) & 1], (uint64_t)jn, 128, 128};
            GQ_TRY(schur(jb, jn, gq::NB, jn, 0, jn, false, sn, "chol_update_next", side, &so, true));
            GQ_TRY(cudaEventRecord(ev_N, sn));
            // U2(j) = block column j-2, rows 0 .. j-2 (with its diagonal block), after R(j+1)
            if (jn2 >= 0) {
                GQ_TRY(cudaStreamWaitEvent(sn, ev_R, 0));
                GQ_TRY(schur(jb, jn, gq::NB, jn2, 0, jn2, false, sn, "chol_update_u2", side, nullptr, true));
            }
            GQ_TRY(cudaEventRecord(ev_U2, sn));
            // far stream: R(j) = block columns 0 .. j-3
            if (jn2 > 0) {
                GQ_TRY(cudaStreamWaitEvent(sf, ev_P, 0));
                GQ_TRY(schur(jb, jn2, jn2, 0, 0, 0, true, sf, "chol_update", side, nullptr, true));
                GQ_TRY(cudaEventRecord(ev_R, sf));
            }
        }
        GQ_TRY(inverse_step(j));
    }
    // all streams are done before the caller's stream continues
    GQ_TRY(cudaEventRecord(ev_near, sn));
    GQ_TRY(cudaEventRecord(ev_far, sf));
    GQ_TRY(cudaEventRecord(ev_chain, sc));
    GQ_TRY(cudaEventRecord(ev_inv, si));
    GQ_TRY(cudaStreamWaitEvent(st, ev_near, 0));
    GQ_TRY(cudaStreamWaitEvent(st, ev_far, 0));
    GQ_TRY(cudaStreamWaitEvent(st, ev_chain, 0));
    GQ_TRY(cudaStreamWaitEvent(st, ev_inv, 0));
    return cudaSuccess;
}

}  // namespace gqh
