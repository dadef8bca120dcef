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
//   with the update split three ways: block column j-1 on the critical chain (a stream of
//   the highest priority), then block column j-2 and the rest on a low-priority stream
//   (look-ahead of depth two).
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
//      lane keeps up to date from its own multipliers; the multiplier column reaches the
//      other rows through shared memory, off that chain; 1/L_kk = rsqrt with one Newton step.
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
    float col[2][32];        // multiplier column of the current pivot (double-buffered)
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// A. Factor the 32x32 diagonal block at (k0, k0) with one warp; lane i holds row k0 + i.
// Per pivot k the pivot value is the only shuffle on the dependency chain (each lane keeps
// its own diagonal entry current); the multipliers L_jk reach the other rows through a
// double-buffered column in shared memory (one store, a warp barrier and vector loads).
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
    float dg = 0.f;   // this lane's diagonal entry, kept current with its own multipliers
#pragma unroll
    for (int j = 0; j < 32; ++j) dg = (lane == j) ? a[j] : dg;
    int bad = -1;     // first pivot that is not positive and finite
    float bad_p = 0.f, rr = 0.f;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const float p = __shfl_sync(FULL, dg, k);   // pivot: P_kk after pivots 0..k-1
        const bool pk = p > 0.f && isfinite(p);
        bad_p = (bad < 0 && !pk) ? p : bad_p;
        bad = (bad < 0 && !pk) ? k : bad;
        float r = rsqrtf(p);
        r = r * fmaf(-0.5f * p * r, r, 1.5f);       // one Newton step for 1/sqrt(p)
        const float l = (lane == k) ? p * r : a[k] * r;   // L_kk = sqrt(p); L_ik = P_ik / L_kk
        a[k] = l;
        if (lane > k) dg = fmaf(-l, l, dg);
        rr = (lane == k) ? r : rr;
        if (k < 31) {
            float* cb = S.col[k & 1];
            cb[lane] = l;
            __syncwarp();
#pragma unroll
            for (int j4 = (k + 1) >> 2; j4 < 8; ++j4) {
                const float4 c4 = ld4(&cb[4 * j4]);    // L_jk for j = 4 j4 ..
                if (4 * j4 + 0 > k) a[4 * j4 + 0] = fmaf(-l, c4.x, a[4 * j4 + 0]);
                if (4 * j4 + 1 > k) a[4 * j4 + 1] = fmaf(-l, c4.y, a[4 * j4 + 1]);
                if (4 * j4 + 2 > k) a[4 * j4 + 2] = fmaf(-l, c4.z, a[4 * j4 + 2]);
                if (4 * j4 + 3 > k) a[4 * j4 + 3] = fmaf(-l, c4.w, a[4 * j4 + 3]);
            }
        }
    }
    if (lane == 0 && bad >= 0)
        record_status(isfinite(bad_p) ? GPTQ_ERR_NOT_PD : GPTQ_ERR_NONFINITE, jb + 127 - (k0 + bad));
    S.rinv[k0 + lane] = rr;
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
    return (size_t)(9 * n * n + 2 * n * gq::NB + 64 + n) * sizeof(float);
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
    w.AP_hi = p;   // tf32 split of the next panel, n x 128
    p += n * gq::NB;
    w.AP_lo = p;
    p += n * gq::NB;
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
    // Streams.  The chain stream (highest priority) carries, per block column j,
    //   leaf(j) -> panel(j): R_{0:j,j} = A_{0:j,j} X_jj^T
    //           -> block column j-1 updated by panel j (and the next panel's tf32 split).
    // The far stream takes the rest of panel j's Schur update: first block column j-2 (u2),
    // then everything left of it (rest).  Block column j-1 has received, before its update by
    // panel j, u2(j+1) and rest(p) for p >= j+2, which the far stream runs in that order, so
    // the chain waits only for u2(j+1).  The inverse stream runs the doubling products.
    FactStreams fs;
    if (!fact_streams(&fs)) return cudaErrorUnknown;
    cudaEvent_t ev_start = fs.ev[0], ev_leaf = fs.ev[1], ev_panel = fs.ev[2], ev_u2 = fs.ev[5],
                ev_far = fs.ev[8], ev_chain = fs.ev[9], ev_inv = fs.ev[10];
    cudaStream_t sc = fs.chain, sf = fs.far, si = fs.inv;
    {
        gqh::TimedScope ts__("zero_lower", st);   // the public U's strictly lower blocks
        const unsigned nb = (unsigned)((d + gq::NB - 1) / gq::NB);
        gq::zero_lower_blocks_kernel<<<dim3(nb, nb), 256, 0, st>>>(U, d);
    }
    GQ_TRY(cudaGetLastError());
    GQ_TRY(cudaEventRecord(ev_start, st));
    GQ_TRY(cudaStreamWaitEvent(sc, ev_start, 0));
    GQ_TRY(cudaStreamWaitEvent(sf, ev_start, 0));
    GQ_TRY(cudaStreamWaitEvent(si, ev_start, 0));
    const int far_ctas = std::max(1, num_sms() - 1);            // leave an SM for the next leaf
    const int inv_ctas = std::max(1, num_sms() / 4);            // the inverse fills in around the chain
    Mat rh{w.RS_hi, N, N, N}, rl{w.RS_lo, N, N, N};
    Mat xh{w.U_hi, N, N, N}, xl{w.U_lo, N, N, N};
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
        if (narrow) return launch_gemm<gq::KIND_TF32X3, 4, 32, 2>(rh, rl, uth, utl, o, p, 1, si, "inv_bu", inv_ctas, true);
        return launch_gemm<gq::KIND_TF32X3, 2, 128, 4>(rh, rl, uth, utl, o, p, 1, si, "inv_bu", inv_ctas, true);
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
        // the pairs that contain block 0 are the tail after the last leaf: all SMs
        const int cap = r0 == 0 ? 0 : inv_ctas;
        const bool narrow = 4 * (s_ / gq::NB) * ((cs + gq::NB - 1) / gq::NB) <= num_sms();
        if (narrow) return launch_gemm<gq::KIND_TF32X3, 4, 32, 2>(xh, xl, tth, ttl, o, p, 1, si, "inv_ub", cap, true);
        return launch_gemm<gq::KIND_TF32X3, 2, 128, 4>(xh, xl, tth, ttl, o, p, 1, si, "inv_ub", cap, true);
    };
    // the inverse work that becomes possible once leaf(j) and panel(j) are done (event ev)
    auto inverse_step = [&](int j, cudaEvent_t ev) -> cudaError_t {
        const long long jb = (long long)j * gq::NB;
        GQ_TRY(cudaStreamWaitEvent(si, ev, 0));
        {
            gqh::TimedScope ts__("chol_diag_out", si);
            gq::chol_diag_out_kernel<<<1, 512, dout_smem, si>>>(w.U_hi, w.U_lo, w.UT_hi, w.UT_lo, U, n, d, j);
        }
        GQ_TRY(cudaGetLastError());
        for (long long s_ = gq::NB; s_ < n; s_ *= 2)   // pairs whose a-half starts at block j
            if (jb % (2 * s_) == 0 && jb + s_ < n) GQ_TRY(inv_ub(s_, jb, std::min(s_, n - jb - s_)));
        for (long long s_ = gq::NB; s_ < n; s_ *= 2)   // pairs whose c-half starts at block j
            if (jb >= s_ && (jb - s_) % (2 * s_) == 0) GQ_TRY(inv_bu(s_, jb - s_, std::min(s_, n - jb)));
        return cudaSuccess;
    };
    bool u2_pending = false;
    for (int j = T - 1; j >= 0; --j) {
        const int jb = j * gq::NB;
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
            GQ_TRY(inverse_step(0, ev_leaf));
            break;
        }
        if (j == T - 1) {   // later panels are split by the previous update's epilogue
            gqh::TimedScope ts__("split_panel", sc);
            gq::split_panel_kernel<<<(unsigned)std::min<long long>((jb * 128LL + 255) / 256, 4096), 256, 0, sc>>>(
                w.A, n, jb, jb, w.AP_hi, w.AP_lo);
            GQ_TRY(cudaGetLastError());
        }
        {   // panel: RS[0:jb, jb:jb+128] = AP * X^T, X = U block (row-major split)
            gq::GemmArgs p = gemm_args(jb, gq::NB, gq::NB);
            p.b_row0 = jb;
            p.b_col0 = jb;
            p.s_col0 = jb;
            EpiMats o;
            o.s_hi = Mat{w.RS_hi, N, N, N};
            o.s_lo = Mat{w.RS_lo, N, N, N};
            Mat ah{w.AP_hi, (uint64_t)jb, 128, 128}, al{w.AP_lo, (uint64_t)jb, 128, 128};
            GQ_TRY((launch_gemm<gq::KIND_TF32X3, 4, 32, 2>(ah, al, xh, xl, o, p, 1, sc, "chol_panel", 0,
                                                        j == T - 1)));
        }
        const int jn = jb - gq::NB;    // first column of block column j-1
        const int jn2 = jn - gq::NB;   // first column of block column j-2
        GQ_TRY(cudaEventRecord(ev_panel, sc));
        const bool waited = u2_pending;
        if (u2_pending) GQ_TRY(cudaStreamWaitEvent(sc, ev_u2, 0));
        {   // block column j-1: A[0:jb, jn:jb] -= RS_panel RS_panel[jn:jb]^T, plus the next panel's split
            gq::GemmArgs p = gemm_args(jb, gq::NB, gq::NB);
            p.a_col0 = jb;
            p.b_row0 = jn;
            p.b_col0 = jb;
            p.alpha = -1.f;
            p.beta = 1.f;
            p.write_c = 1;
            p.c_col0 = jn;
            EpiMats o;
            o.c = Mat{w.A, N, N, N};
            if (j >= 2) {   // tiles above the diagonal block write the next panel's tf32 split
                p.s_mt_lim = j - 1;
                o.s_hi = Mat{w.AP_hi, (uint64_t)jn, 128, 128};
                o.s_lo = Mat{w.AP_lo, (uint64_t)jn, 128, 128};
            }
            GQ_TRY((launch_gemm<gq::KIND_TF32X3, 4, 32, 2>(rh, rl, rh, rl, o, p, 1, sc, "chol_update_next", 0,
                                                        waited)));
        }
        u2_pending = false;
        if (j >= 2) {   // far stream: block column j-2, then the rest
            GQ_TRY(cudaStreamWaitEvent(sf, ev_panel, 0));
            {   // u2: A[0:jn, jn2:jn] -= RS_panel RS_panel[jn2:jn]^T
                gq::GemmArgs p = gemm_args(jn, gq::NB, gq::NB);
                p.a_col0 = jb;
                p.b_row0 = jn2;
                p.b_col0 = jb;
                p.alpha = -1.f;
                p.beta = 1.f;
                p.write_c = 1;
                p.c_col0 = jn2;
                EpiMats o;
                o.c = Mat{w.A, N, N, N};
                GQ_TRY((launch_gemm<gq::KIND_TF32X3, 4, 32, 2>(rh, rl, rh, rl, o, p, 1, sf, "chol_update_u2",
                                                            far_ctas, true)));
            }
            GQ_TRY(cudaEventRecord(ev_u2, sf));
            u2_pending = true;
            if (j >= 3) {   // rest: A[0:jn2, 0:jn2] -= RS RS^T (upper tiles)
                gq::GemmArgs p = gemm_args(jn2, jn2, gq::NB);
                p.a_col0 = jb;
                p.b_col0 = jb;
                p.triangular = 1;
                p.alpha = -1.f;
                p.beta = 1.f;
                p.write_c = 1;
                EpiMats o;
                o.c = Mat{w.A, N, N, N};
                GQ_TRY((launch_gemm<gq::KIND_TF32X3, 2, 128, 4>(rh, rl, rh, rl, o, p, 1, sf, "chol_update",
                                                       far_ctas, true)));
            }
        }
        GQ_TRY(inverse_step(j, ev_panel));
    }
    // all streams are done before the caller's stream continues
    GQ_TRY(cudaEventRecord(ev_far, sf));
    GQ_TRY(cudaEventRecord(ev_chain, sc));
    GQ_TRY(cudaEventRecord(ev_inv, si));
    GQ_TRY(cudaStreamWaitEvent(st, ev_far, 0));
    GQ_TRY(cudaStreamWaitEvent(st, ev_chain, 0));
    GQ_TRY(cudaStreamWaitEvent(st, ev_inv, 0));
    return cudaSuccess;
}

}  // namespace gqh
