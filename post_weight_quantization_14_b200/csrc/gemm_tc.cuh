// tcgen05 tensor-core GEMM with TMA-fed, 128-byte-swizzled K-major operands and an
// fp32 accumulator in tensor memory.
//
//   D[i, j] = sum_k A[i, k] * B[j, k]      (i < M, j < N, k in the tile's K range)
//   out     = alpha * D + beta * C[i, j]   -> written to any of: C (row-major fp32),
//             S_hi/S_lo (row-major tf32 split of out), T_hi/T_lo (transposed tf32 split),
//             and, for symmetric updates, the mirrored C[j, i].
//
// KIND_BF16   : A, B bf16 (kind::f16), one MMA per 16-element K step.
// KIND_TF32X3 : A = A_hi + A_lo and B = B_hi + B_lo given as two tf32 arrays each;
//               three MMAs per 8-element K step (hi*hi + hi*lo + lo*hi), which keeps
//               about fp32 accuracy on the tf32 tensor pipe.
//
// One 128 x BN output tile per CTA; warp 0 issues TMA, warp 1 issues MMAs, warps
// 2..5 read the accumulator from tensor memory and run the epilogue.  The epilogue is
// TMA-based: for C -= A B^T updates the C tile is fetched by TMA while the mainloop
// runs (PREFETCH_C), and every output is written as 32x32 boxes staged in
// 128-byte-swizzled shared memory and stored by TMA, double-buffered per warp, so the
// HBM traffic of the epilogue runs asynchronously.  Tiles on the diagonal of a
// mirrored (symmetric) output take a register path that writes j >= i and mirrors
// it exactly.  Every wait is bounded (GPTQ_ERR_TIMEOUT).  No TMA multicast.
//
// Outputs are clipped by the extents of their tensor maps; every caller keeps M and
// N either multiples of the tile or equal to the remaining extent of the output.
#pragma once
#include "common.cuh"

namespace gq {

enum : int { KIND_BF16 = 0, KIND_TF32X3 = 1 };

struct GemmArgs {
    int M, N, K;
    int a_row0, a_col0, a_zrow, a_zcol;   // A(i,k) at map (x = a_col0 + k, y = a_row0 + i)
    int b_row0, b_col0, b_zrow, b_zcol;   // B(j,k) at map (x = b_col0 + k, y = b_row0 + j)
    int tiles_m, tiles_n;
    int triangular;   // enumerate only tiles with nt >= mt (BM == BN)
    int k_from_m0;    // K range of a tile starts at its m0 (A upper triangular in (i,k))
    int k_to_n1;      // K range of a tile ends at n0 + BN (B zero for k > j)
    float alpha, beta;
    float* C;
    long long ldc;
    int c_row0, c_col0, c_zrow, c_zcol;
    int write_c;
    int c_lim_rows, c_lim_cols;  // if > 0: C positions at or beyond these are neither read nor written
    int mirror;       // also write C[j, i] for tiles above the diagonal
    float* S_hi;
    float* S_lo;
    long long lds;
    int s_row0, s_col0, s_zrow, s_zcol;
    int s_tile_n;     // if > 0: S written only by tiles with nt == s_tile_n and mt < nt
    float* T_hi;
    float* T_lo;
    long long ldt;
    int t_row0, t_col0, t_zrow, t_zcol;
};

constexpr int kEpiLd = 33;
constexpr int kEpiBytes = 4 * 32 * kEpiLd * 4;

template <int KIND>
struct GemmCfg {
    static constexpr int BM = 128;
    static constexpr int KT = (KIND == KIND_BF16) ? 64 : 32;  // K elements per stage (128 bytes)
    static constexpr int NOPS = (KIND == KIND_BF16) ? 1 : 2;
};

__device__ __forceinline__ void tile_coords(const GemmArgs& p, int t, int& mt, int& nt) {
    if (!p.triangular) {
        mt = t / p.tiles_n;
        nt = t % p.tiles_n;
        return;
    }
    int row = 0;
    int rem = t;
    while (row < p.tiles_m) {
        int cnt = p.tiles_n - row;
        if (rem < cnt) break;
        rem -= cnt;
        ++row;
    }
    mt = row;
    nt = row + rem;
}

__device__ __forceinline__ void store_split(float* hi, float* lo, long long idx, float v) {
    float h, l;
    split_tf32(v, h, l);
    hi[idx] = h;
    lo[idx] = l;
}

constexpr int kBoxBytes = 32 * 32 * 4;   // one 32x32 fp32 box, 128-byte rows

// Byte offset of element (row, col) in a 128-byte-swizzled 32x32 fp32 box.
__device__ __forceinline__ uint32_t box_off(int row, int col) {
    return (uint32_t)(row * 128 + ((((col >> 2) ^ (row & 7))) << 4) + (col & 3) * 4);
}
// Thread `row` writes its 32 values as one row of the box.
__device__ __forceinline__ void box_put_row(uint8_t* box, int row, const float (&v)[32]) {
#pragma unroll
    for (int c4 = 0; c4 < 8; ++c4)
        *reinterpret_cast<float4*>(box + row * 128 + ((c4 ^ (row & 7)) << 4)) =
            make_float4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
}
// Thread `col` writes its 32 values as one column of the box (transposed output).
__device__ __forceinline__ void box_put_col(uint8_t* box, int col, const float (&v)[32]) {
#pragma unroll
    for (int t = 0; t < 32; ++t) *reinterpret_cast<float*>(box + box_off(t, col)) = v[t];
}

template <int KIND, int BN, int STAGES, bool PREFETCH_C>
__global__ void __launch_bounds__(192, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mA2,
                   const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mB2,
                   const __grid_constant__ CUtensorMap mC, const __grid_constant__ CUtensorMap mS1,
                   const __grid_constant__ CUtensorMap mS2, const __grid_constant__ CUtensorMap mT1,
                   const __grid_constant__ CUtensorMap mT2, const GemmArgs p) {
    using Cfg = GemmCfg<KIND>;
    constexpr int BM = Cfg::BM, KT = Cfg::KT, NOPS = Cfg::NOPS;
    constexpr int A_BYTES = BM * 128;
    constexpr int B_BYTES = BN * 128;
    constexpr int STAGE_BYTES = NOPS * (A_BYTES + B_BYTES);
    constexpr uint32_t TMEM_COLS = BN;  // power of two >= 32
    static_assert(BN == 128 || BN == 256, "BN");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    constexpr int CIN_BYTES = PREFETCH_C ? BM * BN * 4 : 0;
    uint8_t* cin = smem + STAGES * STAGE_BYTES;                       // prefetched C boxes
    float* epi = reinterpret_cast<float*>(cin + CIN_BYTES);           // 4 warps x 32 x 33
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(epi) + kEpiBytes);
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* acc_bar = empty_bar + STAGES;
    uint64_t* cin_bar = acc_bar + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cin_bar + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int mt, nt;
    tile_coords(p, blockIdx.x, mt, nt);
    const int z = blockIdx.z;
    const int m0 = mt * BM, n0 = nt * BN;
    const int kbeg = p.k_from_m0 ? m0 : 0;
    const int kend = p.k_to_n1 ? min(p.K, n0 + BN) : p.K;
    const int nk = kend > kbeg ? (kend - kbeg + KT - 1) / KT : 0;
    const long long where = ((long long)blockIdx.z << 32) | (long long)blockIdx.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(acc_bar, 1);
        mbar_init(cin_bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {
        prefetch_tmap(&mA);
        prefetch_tmap(&mB);
        if (NOPS == 2) {
            prefetch_tmap(&mA2);
            prefetch_tmap(&mB2);
        }
        const int ax = p.a_col0 + z * p.a_zcol, ay = p.a_row0 + z * p.a_zrow + m0;
        const int bx = p.b_col0 + z * p.b_zcol, by = p.b_row0 + z * p.b_zrow + n0;
        if (PREFETCH_C && p.beta != 0.f) {   // the C tile, as 32x32 boxes, while the mainloop runs
            prefetch_tmap(&mC);
            mbar_arrive_expect_tx(cin_bar, CIN_BYTES);
            const int cx = p.c_col0 + z * p.c_zcol + n0, cy = p.c_row0 + z * p.c_zrow + m0;
            for (int q = 0; q < 4; ++q)
                for (int c = 0; c < BN / 32; ++c)
                    tma_load_2d(cin + (q * (BN / 32) + c) * kBoxBytes, &mC, cin_bar, cx + 32 * c, cy + 32 * q);
        }
        for (int kt = 0; kt < nk; ++kt) {
            const int s = kt % STAGES;
            const uint32_t it = kt / STAGES;
            if (!mbar_wait(&empty_bar[s], (it & 1) ^ 1, where)) break;
            uint8_t* st = smem + s * STAGE_BYTES;
            mbar_arrive_expect_tx(&full_bar[s], STAGE_BYTES);
            const int k = kbeg + kt * KT;
            tma_load_2d(st, &mA, &full_bar[s], ax + k, ay);
            if (NOPS == 2) tma_load_2d(st + A_BYTES, &mA2, &full_bar[s], ax + k, ay);
            tma_load_2d(st + NOPS * A_BYTES, &mB, &full_bar[s], bx + k, by);
            if (NOPS == 2) tma_load_2d(st + NOPS * A_BYTES + B_BYTES, &mB2, &full_bar[s], bx + k, by);
        }
    } else if (warp == 1 && lane == 0) {
        constexpr uint32_t idesc = make_idesc(KIND == KIND_BF16 ? 1u : 2u, BM, BN);
        bool ok = true;
        for (int kt = 0; kt < nk && ok; ++kt) {
            const int s = kt % STAGES;
            const uint32_t it = kt / STAGES;
            if (!mbar_wait(&full_bar[s], it & 1, where)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t st = smem_u32(smem + s * STAGE_BYTES);
            const uint32_t a_hi = st, a_lo = st + A_BYTES;
            const uint32_t b_hi = st + NOPS * A_BYTES, b_lo = b_hi + B_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t off = kk * 32;
                const uint32_t acc0 = (kt > 0 || kk > 0) ? 1u : 0u;
                if (KIND == KIND_BF16) {
                    umma_bf16(tmem, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_hi + off), idesc,
                              acc0);
                } else {
                    umma_tf32(tmem, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_hi + off), idesc,
                              acc0);
                    umma_tf32(tmem, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_lo + off), idesc,
                              1u);
                    umma_tf32(tmem, desc_sw128_kmajor(a_lo + off), desc_sw128_kmajor(b_hi + off), idesc,
                              1u);
                }
            }
            umma_commit(&empty_bar[s]);
        }
        umma_commit(acc_bar);
    } else if (warp >= 2) {
        const bool ok = mbar_wait(acc_bar, 0, where);
        tc_fence_after();
        const bool diag_mirror = p.mirror && nt == mt;
        if (!diag_mirror) {
            // TMA epilogue
            const int q = warp & 3;
            const bool mirror = p.mirror && nt > mt;
            const bool has_c = p.write_c != 0, has_t = p.T_hi != nullptr;
            const bool has_s = p.S_hi != nullptr && (p.s_tile_n <= 0 || (nt == p.s_tile_n && mt < nt));
            const int nkinds = (has_c ? 1 : 0) + (has_s ? 2 : 0) + (has_t ? 2 : 0) + (mirror ? 1 : 0);
            const int kc = 0, ks = kc + (has_c ? 1 : 0), kt = ks + (has_s ? 2 : 0), km = kt + (has_t ? 2 : 0);
            const bool use_cin = PREFETCH_C && p.beta != 0.f;
            bool cin_ok = true;
            if (use_cin) cin_ok = mbar_wait(cin_bar, 0, where);
            const int zc_x = p.c_col0 + z * p.c_zcol, zc_y = p.c_row0 + z * p.c_zrow;
            const int zs_x = p.s_col0 + z * p.s_zcol, zs_y = p.s_row0 + z * p.s_zrow;
            const int zt_x = p.t_col0 + z * p.t_zcol, zt_y = p.t_row0 + z * p.t_zrow;
            const int iy = m0 + 32 * q;   // first accumulator row of this warp
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                const int j0 = n0 + c * 32;
                if (j0 >= p.N) break;
                uint32_t r[32];
                if (nk > 0 && ok) {
                    tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(c * 32), r);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int t = 0; t < 32; ++t) r[t] = 0u;
                }
                float out[32];
#pragma unroll
                for (int t = 0; t < 32; ++t) out[t] = p.alpha * __uint_as_float(r[t]);
                if (use_cin && cin_ok) {
                    const uint8_t* box = cin + (q * (BN / 32) + c) * kBoxBytes;
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 v = *reinterpret_cast<const float4*>(box + lane * 128 + ((c4 ^ (lane & 7)) << 4));
                        out[4 * c4 + 0] = fmaf(p.beta, v.x, out[4 * c4 + 0]);
                        out[4 * c4 + 1] = fmaf(p.beta, v.y, out[4 * c4 + 1]);
                        out[4 * c4 + 2] = fmaf(p.beta, v.z, out[4 * c4 + 2]);
                        out[4 * c4 + 3] = fmaf(p.beta, v.w, out[4 * c4 + 3]);
                    }
                }
                // output boxes of this chunk live in the (now idle) stage buffers, two slots per warp
                uint8_t* ob = smem + ((q * 2 + (c & 1)) * nkinds) * kBoxBytes;
                if (c >= 2) {
                    if (lane == 0) bulk_wait_read_1();
                    __syncwarp();
                }
                if (has_c) box_put_row(ob + kc * kBoxBytes, lane, out);
                if (has_s || has_t) {
                    float hi[32], lo[32];
#pragma unroll
                    for (int t = 0; t < 32; ++t) split_tf32(out[t], hi[t], lo[t]);
                    if (has_s) {
                        box_put_row(ob + ks * kBoxBytes, lane, hi);
                        box_put_row(ob + (ks + 1) * kBoxBytes, lane, lo);
                    }
                    if (has_t) {
                        box_put_col(ob + kt * kBoxBytes, lane, hi);
                        box_put_col(ob + (kt + 1) * kBoxBytes, lane, lo);
                    }
                }
                if (mirror) box_put_col(ob + km * kBoxBytes, lane, out);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (has_c) tma_store_2d(&mC, ob + kc * kBoxBytes, zc_x + j0, zc_y + iy);
                    if (has_s) {
                        tma_store_2d(&mS1, ob + ks * kBoxBytes, zs_x + j0, zs_y + iy);
                        tma_store_2d(&mS2, ob + (ks + 1) * kBoxBytes, zs_x + j0, zs_y + iy);
                    }
                    if (has_t) {
                        tma_store_2d(&mT1, ob + kt * kBoxBytes, zt_x + iy, zt_y + j0);
                        tma_store_2d(&mT2, ob + (kt + 1) * kBoxBytes, zt_x + iy, zt_y + j0);
                    }
                    if (mirror) tma_store_2d(&mC, ob + km * kBoxBytes, zc_x + iy, zc_y + j0);
                    bulk_commit();
                }
            }
            if (lane == 0) bulk_wait_all();
            __syncwarp();
        } else {
            // Register path for diagonal tiles of mirrored outputs: write j >= i and its exact mirror.
            const int q = warp & 3;
            float* tile = epi + q * 32 * kEpiLd;
            const int rbase = m0 + q * 32;
            const bool mirror = false;
            const bool diag_tile = true;   // write j >= i only, mirrored below
            const long long zc_row = p.c_row0 + (long long)z * p.c_zrow, zc_col = p.c_col0 + (long long)z * p.c_zcol;
            const long long zs_row = p.s_row0 + (long long)z * p.s_zrow, zs_col = p.s_col0 + (long long)z * p.s_zcol;
            const long long zt_row = p.t_row0 + (long long)z * p.t_zrow, zt_col = p.t_col0 + (long long)z * p.t_zcol;
            const bool pass2 = (p.T_hi != nullptr) || mirror || diag_tile;
    #pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                const int j0 = n0 + c * 32;
                if (j0 >= p.N) break;
                uint32_t r[32];
                if (nk > 0 && ok) {
                    tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(c * 32), r);
                    tmem_ld_wait();
                } else {
    #pragma unroll
                    for (int t = 0; t < 32; ++t) r[t] = 0u;
                }
    #pragma unroll
                for (int t = 0; t < 32; ++t) tile[lane * kEpiLd + t] = __uint_as_float(r[t]);
                __syncwarp();
                {   // pass 1: lane = column; all 32 row loads of C are issued before any use
                    const int j = j0 + lane;
                    const bool col_ok = j < p.N;
                    const long long ac = zc_col + j;
                    const bool c_col_ok = col_ok && (p.c_lim_cols <= 0 || ac < p.c_lim_cols);
                    const int nrows = max(0, min(32, p.M - rbase));
                    float cv[32];
                    if (p.beta != 0.f) {
    #pragma unroll
                        for (int rr = 0; rr < 32; ++rr) {
                            const long long ar = zc_row + rbase + rr;
                            const bool c_ok = rr < nrows && c_col_ok && (p.c_lim_rows <= 0 || ar < p.c_lim_rows);
                            cv[rr] = c_ok ? p.C[ar * p.ldc + ac] : 0.f;
                        }
                    } else {
    #pragma unroll
                        for (int rr = 0; rr < 32; ++rr) cv[rr] = 0.f;
                    }
    #pragma unroll
                    for (int rr = 0; rr < 32; ++rr) {
                        const int i = rbase + rr;
                        const long long ar = zc_row + i;
                        const bool c_ok = rr < nrows && c_col_ok && (p.c_lim_rows <= 0 || ar < p.c_lim_rows);
                        const float out = fmaf(p.beta, cv[rr], p.alpha * tile[rr * kEpiLd + lane]);
                        if (p.write_c && c_ok && (!diag_tile || j >= i)) p.C[ar * p.ldc + ac] = out;
                        if (p.S_hi && col_ok && rr < nrows) store_split(p.S_hi, p.S_lo, (zs_row + i) * p.lds + zs_col + j, out);
                        tile[rr * kEpiLd + lane] = out;
                    }
                }
                __syncwarp();
                if (pass2) {   // pass 2: lane = row
                    const int i = rbase + lane;
                    const bool row_ok = i < p.M;
    #pragma unroll 4
                    for (int t = 0; t < 32; ++t) {
                        const int jj = j0 + t;
                        if (jj >= p.N) break;
                        const float out = tile[lane * kEpiLd + t];
                        if (row_ok && p.T_hi) store_split(p.T_hi, p.T_lo, (zt_row + jj) * p.ldt + zt_col + i, out);
                        if (row_ok && (mirror || (diag_tile && jj > i))) p.C[(zc_row + jj) * p.ldc + zc_col + i] = out;
                    }
                }
                __syncwarp();
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int KIND, int BN, int STAGES, bool PREFETCH_C>
constexpr int gemm_smem_bytes() {
    return STAGES * GemmCfg<KIND>::NOPS * (128 * 128 + BN * 128) + (PREFETCH_C ? 128 * BN * 4 : 0) + kEpiBytes +
           1024 + 256;
}

}  // namespace gq

namespace gqh {

// One operand of the GEMM: a row-major matrix [rows, cols] (K is the column index).
struct Mat {
    const void* ptr;
    uint64_t rows, cols, ld;  // elements
};

// Output matrices of the epilogue (ptr == nullptr: not written).  C is also the
// matrix read when beta != 0 and the target of mirrored writes.
struct EpiMats {
    Mat c{nullptr, 0, 0, 0}, s_hi{nullptr, 0, 0, 0}, s_lo{nullptr, 0, 0, 0}, t_hi{nullptr, 0, 0, 0},
        t_lo{nullptr, 0, 0, 0};
};

inline bool make_out_map(CUtensorMap* map, const Mat& m, const CUtensorMap& fallback) {
    if (!m.ptr) {
        *map = fallback;
        return true;
    }
    return make_tmap_2d(map, m.ptr, 4, m.rows, m.cols, m.ld, 32, 32);
}

// Launch D = A B^T with the given epilogue.  For KIND_TF32X3 a2/b2 are the lo parts.
// PREFETCH_C is required when p.beta != 0.
template <int KIND, int BN, int STAGES, bool PREFETCH_C>
cudaError_t launch_gemm(const Mat& a, const Mat& a2, const Mat& b, const Mat& b2, const EpiMats& o, gq::GemmArgs p,
                        int batch, cudaStream_t stream, const char* name) {
    using Cfg = gq::GemmCfg<KIND>;
    const int eb = (KIND == gq::KIND_BF16) ? 2 : 4;
    if (p.beta != 0.f && !PREFETCH_C) return cudaErrorInvalidValue;
    CUtensorMap ma, ma2, mb, mb2, mc, ms1, ms2, mt1, mt2;
    if (!make_tmap_2d(&ma, a.ptr, eb, a.rows, a.cols, a.ld, 128, Cfg::KT)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&mb, b.ptr, eb, b.rows, b.cols, b.ld, BN, Cfg::KT)) return cudaErrorInvalidValue;
    if (KIND == gq::KIND_TF32X3) {
        if (!make_tmap_2d(&ma2, a2.ptr, eb, a2.rows, a2.cols, a2.ld, 128, Cfg::KT)) return cudaErrorInvalidValue;
        if (!make_tmap_2d(&mb2, b2.ptr, eb, b2.rows, b2.cols, b2.ld, BN, Cfg::KT)) return cudaErrorInvalidValue;
    } else {
        ma2 = ma;
        mb2 = mb;
    }
    if (!make_out_map(&mc, o.c, ma) || !make_out_map(&ms1, o.s_hi, ma) || !make_out_map(&ms2, o.s_lo, ma) ||
        !make_out_map(&mt1, o.t_hi, ma) || !make_out_map(&mt2, o.t_lo, ma))
        return cudaErrorInvalidValue;
    p.C = static_cast<float*>(const_cast<void*>(o.c.ptr));
    p.ldc = (long long)o.c.ld;
    p.S_hi = static_cast<float*>(const_cast<void*>(o.s_hi.ptr));
    p.S_lo = static_cast<float*>(const_cast<void*>(o.s_lo.ptr));
    p.lds = (long long)o.s_hi.ld;
    p.T_hi = static_cast<float*>(const_cast<void*>(o.t_hi.ptr));
    p.T_lo = static_cast<float*>(const_cast<void*>(o.t_lo.ptr));
    p.ldt = (long long)o.t_hi.ld;
    // output boxes (two slots per warp) must fit in the stage buffers they reuse
    const int kinds = (p.write_c ? 1 : 0) + (p.S_hi ? 2 : 0) + (p.T_hi ? 2 : 0) + (p.mirror ? 1 : 0);
    if (4 * 2 * kinds * gq::kBoxBytes > STAGES * Cfg::NOPS * (128 * 128 + BN * 128)) return cudaErrorInvalidValue;
    p.tiles_m = (p.M + 127) / 128;
    p.tiles_n = (p.N + BN - 1) / BN;
    long long tiles = p.triangular ? (long long)p.tiles_m * (p.tiles_m + 1) / 2
                                   : (long long)p.tiles_m * p.tiles_n;
    if (tiles <= 0 || batch <= 0) return cudaSuccess;
    constexpr int smem = gq::gemm_smem_bytes<KIND, BN, STAGES, PREFETCH_C>();
    auto kern = gq::tc_gemm_kernel<KIND, BN, STAGES, PREFETCH_C>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)tiles, 1, (unsigned)batch);
    {
        TimedScope ts__(name, stream);
        kern<<<grid, 192, smem, stream>>>(ma, ma2, mb, mb2, mc, ms1, ms2, mt1, mt2, p);
    }
    return cudaGetLastError();
}

inline gq::GemmArgs gemm_args(int M, int N, int K) {
    gq::GemmArgs p{};
    p.M = M;
    p.N = N;
    p.K = K;
    p.alpha = 1.f;
    p.beta = 0.f;
    return p;
}

}  // namespace gqh
