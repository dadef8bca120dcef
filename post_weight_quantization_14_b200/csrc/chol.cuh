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
    // each thread adds its entries i = tid, tid + blockDim, ... in that order; eight loads in
    // flight per step
    for (long long i0 = threadIdx.x; i0 < d; i0 += 8LL * blockDim.x) {
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const long long i = i0 + (long long)q * blockDim.x;
            v[q] = i < d ? H[i * d + i] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (i0 + (long long)q * blockDim.x < d) s += (double)v[q];
    }
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
                                                        const float* __restrict__ lam, float* __restrict__ A,
                                                        float* __restrict__ RS_hi, float* __restrict__ RS_lo,
                                                        float* __restrict__ U, int* __restrict__ ctr, int nctr) {
    // a 1-D grid of T*T CTAs, the T diagonal blocks first: their sub-tile passes are the
    // longest, so they start before the copies and the zeroing rather than trail them
    const int T = (int)(n / NB);
    const int b = blockIdx.x;
    int bi, bj;
    if (b < T) {
        bi = bj = b;
    } else {
        const int o = b - T;
        bi = o / (T - 1);
        bj = o % (T - 1);
        if (bj >= bi) ++bj;
    }
    const long long r0 = (long long)bi * NB, c0 = (long long)bj * NB;
    if (bi > bj) {   // the public U's strictly lower blocks are zero (d % 4 == 0)
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int e = threadIdx.x; e < NB * NB / 4; e += blockDim.x) {
            const long long i = r0 + (e >> 5), j = c0 + (e & 31) * 4;
            if (i < d && j < d) *reinterpret_cast<float4*>(U + i * d + j) = z;
        }
        return;
    }
    if (bi == 0 && bj == 0)   // the factorization's dependency counters start at zero
        for (int e = threadIdx.x; e < nctr; e += blockDim.x) ctr[e] = 0;
    const float l = lam[0];
    if (bi < bj) {
        const bool last = c0 + NB == n;   // the first panel: also its tf32 split
        constexpr int PER = NB * NB / 4 / 256;   // float4s per thread, all loads issued first
        float4 v[PER];
        long long bad = -1;
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            const int e = threadIdx.x + 256 * q;
            const long long i = r0 + (e >> 5), j = c0 + (e & 31) * 4;
            v[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < d && j < d) v[q] = *reinterpret_cast<const float4*>(H + i * d + j);   // d % 4 == 0
        }
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            const int e = threadIdx.x + 256 * q;
            const long long i = r0 + (e >> 5), j = c0 + (e & 31) * 4;
            if (bad < 0 && !(isfinite(v[q].x) && isfinite(v[q].y) && isfinite(v[q].z) && isfinite(v[q].w)))
                bad = i * d + j;
            *reinterpret_cast<float4*>(A + i * n + j) = v[q];
            if (last) {
                float4 h, lo;
                split_tf32(v[q].x, h.x, lo.x);
                split_tf32(v[q].y, h.y, lo.y);
                split_tf32(v[q].z, h.z, lo.z);
                split_tf32(v[q].w, h.w, lo.w);
                *reinterpret_cast<float4*>(RS_hi + i * n + j) = h;
                *reinterpret_cast<float4*>(RS_lo + i * n + j) = lo;
            }
        }
        if (bad >= 0) record_status(GPTQ_ERR_NONFINITE, bad);
        return;
    }
    // diagonal block: A[i][j] = H[min(i,j)][max(i,j)], by 32x32 sub-tiles of the upper
    // triangle read row by row and written both ways through shared memory (a small tile:
    // the static shared memory of the one kernel bounds the residency of every CTA)
    __shared__ float tile[32][33];
    long long bad = -1;
    for (int sbi = 0; sbi < 4; ++sbi)
        for (int sbj = sbi; sbj < 4; ++sbj) {
            __syncthreads();   // the previous sub-tile's readers are done
            for (int t = threadIdx.x; t < 32 * 32; t += blockDim.x) {
                const int rr = t >> 5, cc = t & 31;
                const long long i = r0 + 32 * sbi + rr, j = c0 + 32 * sbj + cc;
                float v = 0.f;
                if (i < d && j < d && (sbi < sbj || rr <= cc)) {
                    v = H[i * d + j];
                    if (bad < 0 && !isfinite(v)) bad = i * d + j;
                }
                tile[rr][cc] = v;
            }
            __syncthreads();
            for (int t = threadIdx.x; t < 32 * 32; t += blockDim.x) {
                const int rr = t >> 5, cc = t & 31;
                const long long i = r0 + 32 * sbi + rr, j = c0 + 32 * sbj + cc;
                float v = (sbi < sbj || rr <= cc) ? tile[rr][cc] : tile[cc][rr];
                if (i == j) v = (i < d) ? v + l : 1.f;
                A[i * n + j] = v;
                if (sbi < sbj) A[(r0 + 32 * sbj + rr) * n + c0 + 32 * sbi + cc] = tile[cc][rr];
            }
        }
    if (bad >= 0) record_status(GPTQ_ERR_NONFINITE, bad);
}

// The damped copy of damp_copy_kernel for the permuted Hessian: A[i][j] =
// H[perm[i]][perm[j]] (+ lambda on the diagonal) for j >= the start of i's 128-block,
// identity padding past d.  One CTA per row of A: it reads one row of H, so every
// sector of H is fetched once.  H must hold both triangles.
__global__ void __launch_bounds__(256) damp_copy_perm_kernel(const float* __restrict__ H,
                                                             const int* __restrict__ perm, long long d, long long n,
                                                             const float* __restrict__ lam, float* __restrict__ A,
                                                             float* __restrict__ RS_hi, float* __restrict__ RS_lo,
                                                             float* __restrict__ U, int* __restrict__ ctr, int nctr) {
    const long long i = blockIdx.x;
    const long long j0 = (i / NB) * NB;
    if (i == 0)   // the factorization's dependency counters start at zero
        for (int e = threadIdx.x; e < nctr; e += blockDim.x) ctr[e] = 0;
    if (i < d)    // the public U's strictly lower blocks: row i left of its block
        for (long long j = threadIdx.x; j < j0; j += blockDim.x) U[i * d + j] = 0.f;
    const long long jl = n - NB;   // the first panel (block column T-1, rows above its block): also split
    float* out = A + i * n;
    if (i >= d) {
        for (long long j = j0 + threadIdx.x; j < n; j += blockDim.x) {
            const float v = (i == j) ? 1.f : 0.f;
            out[j] = v;
            if (i < jl && j >= jl) {
                RS_hi[i * n + j] = v;
                RS_lo[i * n + j] = 0.f;
            }
        }
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
        if (i < jl && j >= jl) {
            float h, q;
            split_tf32(v, h, q);
            RS_hi[i * n + j] = h;
            RS_lo[i * n + j] = q;
        }
    }
}

// Leaf: factor and invert one 128x128 diagonal block of A in shared memory.
// Works on the index-reversed block P = J A_jj J, for which the UL factor becomes an
// ordinary lower Cholesky factor: A_jj = R R^T with R = J L J, and X_jj = R^-1 = J L^-1 J.
//
// Right-looking, blocked by 32 columns, on 256 threads: warp 0 (F) factors the 32x32
// diagonal blocks; warps 1-7 (W) do everything else, around F's chain.  For panel kb
// (columns k0 = 32 kb .. k0 + 31):
//   F: the diagonal block in registers, lane = row (leaf_diag_factor);
//   W: the rows below by substitution (one thread per row), X_kk = L_kk^-1 (one warp), the
//      rank-32 update of the next diagonal block, which releases F for panel kb+1; then,
//      while F factors it, the rest of the trailing update and the inverse's block rows
//      X_ij = -X_ii sum_{k=j}^{i-1} L_ik X_kj (the sums as soon as their inputs exist, the
//      products by X_ii once it is known).
// F and W meet on named barriers (3: F's block done, 4: the next block updated); W syncs
// on barrier 2 among its 224 threads, the whole leaf on barrier 5.
constexpr int LS = NB + 4;   // leaf smem row stride (16-byte aligned rows)
constexpr int LEAF_THREADS = 256;
constexpr int LEAF_W = LEAF_THREADS - 32;   // threads of warps 1-7

struct LeafSmem {
    float P[NB][LS];         // reversed block; lower triangle holds the Schur complement
    float X[NB][LS];         // L^-1 (lower); blocks above the diagonal hold the block-row sums
    float LT[NB][LS];        // L transposed: LT[m][r] = L[r][m]
    float XDT[4][32][36];    // diagonal inverses transposed: XDT[i][m][r] = X_ii[r][m]
    float rinv[NB];          // 1 / L_kk
    float lc[32][32];        // multiplier columns of the diagonal block being factored: lc[k][i] = L_ik
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void nbar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ void nbar_arrive(int id, int n) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void wsync() { nbar_sync(2, LEAF_W); }
// All 256 threads of the leaf (the CTA may have more warps, which take no part).
__device__ __forceinline__ void leaf_sync() { nbar_sync(5, LEAF_THREADS); }

// F: factor the 32x32 diagonal block at (k0, k0); lane i holds row k0 + i.  Per pivot k the
// dependency chain is: the pivot (one shuffle of the diagonal entry that lane k keeps current
// from its own multipliers), 1/sqrt (the hardware reciprocal square root, no refinement: its
// few-ulp error scales the pivot's column by 1 + O(2^-22), a backward error far below the
// fp32 rounding the factorization accumulates anyway), the multipliers, and the
// next column's update with one more shuffle (L_{k+1,k}); the columns past it take the
// multipliers through shared memory, one pivot behind, off that chain.
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
        const float r = rsqrtf(p);   // hardware 1/sqrt (a few ulp): scales column k by 1 + O(2^-22)
        float l = (lane == k) ? p * r : a[k] * r;   // L_kk = sqrt(p); L_ik = P_ik / L_kk
        if (lane < k) l = 0.f;                      // rows above: finished, untouched
        a[k] = (lane >= k) ? l : a[k];
        if (lane > k) dg = fmaf(-l, l, dg);
        rr = (lane == k) ? r : rr;
        if (k < 31) {
            const float c1 = __shfl_sync(FULL, l, k + 1);   // L_{k+1,k}: the next column first
            a[k + 1] = fmaf(-l, c1, a[k + 1]);
            if (k < 30) {
                S.lc[k][lane] = l;
                __syncwarp();
#pragma unroll
                for (int j4 = (k + 2) >> 2; j4 < 8; ++j4) {
                    const float4 c4 = ld4(&S.lc[k][4 * j4]);   // L_jk for j = 4 j4 ..
                    if (4 * j4 + 0 >= k + 2) a[4 * j4 + 0] = fmaf(-l, c4.x, a[4 * j4 + 0]);
                    if (4 * j4 + 1 >= k + 2) a[4 * j4 + 1] = fmaf(-l, c4.y, a[4 * j4 + 1]);
                    if (4 * j4 + 2 >= k + 2) a[4 * j4 + 2] = fmaf(-l, c4.z, a[4 * j4 + 2]);
                    if (4 * j4 + 3 >= k + 2) a[4 * j4 + 3] = fmaf(-l, c4.w, a[4 * j4 + 3]);
                }
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

// W: row i (below the diagonal block): L_i,kb = P_i,kb L_kk^-T by substitution.
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

// W: rank-32 update of the next diagonal block (rows and columns k0+32 .. k0+63, lower
// triangle) by panel kb, on 2x2 micro-tiles (136 threads).
__device__ __forceinline__ void leaf_next_diag_update(LeafSmem& S, int k0, int wt) {
    if (wt >= 136) return;
    int tr = 0, rem = wt;
    while (rem > tr) {
        rem -= tr + 1;
        ++tr;
    }
    const int r0 = k0 + 32 + 2 * tr, c0 = k0 + 32 + 2 * rem;
    float acc[2][2] = {};
#pragma unroll 8
    for (int m = 0; m < 32; ++m) {
        const float2 a = *reinterpret_cast<const float2*>(&S.LT[k0 + m][r0]);
        const float2 b = *reinterpret_cast<const float2*>(&S.LT[k0 + m][c0]);
        acc[0][0] = fmaf(a.x, b.x, acc[0][0]);
        acc[0][1] = fmaf(a.x, b.y, acc[0][1]);
        acc[1][0] = fmaf(a.y, b.x, acc[1][0]);
        acc[1][1] = fmaf(a.y, b.y, acc[1][1]);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) S.P[r0 + i][c0 + j] -= acc[i][j];
}

// W: the rest of the rank-32 trailing update (rows and columns >= k0 + 32, lower
// triangle, without the next diagonal block), 4x4 micro-tiles.
__device__ __forceinline__ void leaf_rest_update(LeafSmem& S, int k0, int wt, int nthreads) {
    const int t0 = k0 + 32, tn = (NB - t0) >> 2;
    const int ntask = tn * (tn + 1) / 2;
    for (int task = wt; task < ntask; task += nthreads) {
        int tr = (int)((sqrtf(8.f * (float)task + 1.f) - 1.f) * 0.5f);
        while (tr * (tr + 1) / 2 > task) --tr;
        while ((tr + 1) * (tr + 2) / 2 <= task) ++tr;
        const int tc = task - tr * (tr + 1) / 2;
        if (tr < 8) continue;   // rows of the next diagonal block: leaf_next_diag_update
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
// x_m = (delta_mj - sum_{m' < m} L_mm' x_m') / L_mm, with 1/L_mm from leaf_diag_factor.
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

// Block row i of X = L^-1, first part: T_ij = sum_{k=j}^{i-1} L_ik X_kj for j < i, kept in
// X's free upper block (j, i).  Needs block rows < i of X and L's block row i.
__device__ __forceinline__ void leaf_band_sums(LeafSmem& S, int i, int wt, int nthreads) {
    for (int task = wt; task < 64 * i; task += nthreads) {
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
}

// Second part: X_ij = -X_ii T_ij (X_ii from leaf_diag_inverse).
__device__ __forceinline__ void leaf_band_mul(LeafSmem& S, int i, int wt, int nthreads) {
    for (int task = wt; task < 64 * i; task += nthreads) {
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
}

// The whole leaf on P (loaded, reversed, and visible to all 256 threads): L in P/LT and
// X = L^-1 in S.X (lower) on return, visible to all 256 threads.
// Optional event trace for profiling builds (GQ_DAG_TRACE defined): %globaltimer stamps,
// 16 slots per leaf (the factorization kernel adds 8 per product task after them).
#ifdef GQ_DAG_TRACE
__device__ unsigned long long* g_dag_trace = nullptr;
#define GQ_LEAF_STAMP(slot)                                                              \
    do {                                                                                 \
        if (g_dag_trace) g_dag_trace[16 * (long long)(jb >> 7) + (slot)] = globaltimer_ns(); \
    } while (0)
#else
#define GQ_LEAF_STAMP(slot) \
    do {                    \
    } while (0)
#endif
__device__ __forceinline__ void leaf_factor(LeafSmem& S, int jb) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp == 0) {
        for (int kb = 0; kb < 4; ++kb) {
            if (kb > 0) nbar_sync(4, LEAF_THREADS);   // W has updated diagonal block kb
            leaf_diag_factor(S, 32 * kb, lane, jb);
            if (lane == 0) GQ_LEAF_STAMP(3 + kb);
            nbar_arrive(3, LEAF_THREADS);             // diagonal block kb factored
        }
    } else {
        // while F factors, warp 4 (which shares F's scheduler) stays out of the way: the
        // work that overlaps a diagonal factor runs on warps 1-3 and 5-7
        const int wt = tid - 32;
        const int wo = warp < 4 ? wt : wt - 32;   // index among warps 1-3, 5-7
        constexpr int NO = LEAF_W - 32;
        for (int kb = 0; kb < 4; ++kb) {
            const int k0 = 32 * kb;
            nbar_sync(3, LEAF_THREADS);
            if (wt < NB - k0 - 32) leaf_panel_solve(S, k0, k0 + 32 + wt);   // rows below, one each
            else if (warp == 7) leaf_diag_inverse(S, kb, lane);
            wsync();
            if (kb < 3) {
                leaf_next_diag_update(S, k0, wt);
                nbar_arrive(4, LEAF_THREADS);
                if (warp != 4) leaf_rest_update(S, k0, wo, NO);
            }
            if (kb == 3) {   // F is done: all of W
                leaf_band_mul(S, kb, wt, LEAF_W);
                wsync();
            } else if (kb >= 1) {
                if (warp != 4) leaf_band_mul(S, kb, wo, NO);
                wsync();
            }
            if (kb < 3 && warp != 4) leaf_band_sums(S, kb + 1, wo, NO);
        }
    }
    leaf_sync();
}

}  // namespace gq
