// Persistent tcgen05 tensor-core GEMM with TMA-fed, 128-byte-swizzled K-major
// operands and fp32 accumulators in tensor memory.
//
//   D[i, j] = sum_k A[i, k] * B[j, k]      (i < M, j < N, k in the tile's K range)
//   out     = alpha * D + beta * C[i, j]   -> written to C (row-major fp32) and, for
//             symmetric products, also to the mirrored C[j, i].
//
// KIND_BF16   : A, B bf16 (kind::f16), one MMA per 16-element K step.
// KIND_TF32X3 : A = A_hi + A_lo and B = B_hi + B_lo given as two tf32 arrays each;
//               three MMAs per 8-element K step (hi*hi + hi*lo + lo*hi), which keeps
//               about fp32 accuracy on the tf32 tensor pipe.
// KIND_BF16X3 : the same three-product split with bf16 parts (hi = bf16(x),
//               lo = bf16(x - hi): 16 significant bits), one 16-element K step per MMA
//               triple, at the bf16 rate and half the operand bytes of KIND_TF32X3.
//
// Segmented accumulation (SEG > 0): the tensor pipe's fp32 accumulation error grows with
// the number of MMAs accumulated in place, so every SEG MMA k-steps the accumulator is
// handed to the epilogue, which adds it into a running sum in tensor memory with
// round-to-nearest fp32 adds; for the tf32 kinds the small cross products go to an
// accumulator of their own, so segments hold hi*hi products only.
//
// Persistent and warp-specialised: each CTA walks tiles blockIdx.x, +gridDim.x, ...
// Warp 0 issues TMA into a ring of STAGES operand buffers that runs across tiles;
// warp 1 issues MMAs into one of two TMEM accumulators (tile parity), so the epilogue
// of one tile overlaps the mainloop of the next; the epilogue warps (eight for 128-wide
// tiles: two per TMEM lane quadrant, two 32-column chunks each; four otherwise) own 32
// accumulator rows each, load their C chunks by TMA while the MMAs run when beta != 0,
// and write
// every output 32x32 block through a 128-byte-swizzled staging box in shared memory with
// coalesced 16-byte stores (no store-completion waits inside a tile).  Tiles on the
// diagonal of a mirrored (symmetric) output take a register path that writes j >= i and
// mirrors it exactly.  Every wait is bounded (GPTQ_ERR_TIMEOUT).  No TMA multicast.
//
// Outputs are clipped by their matrices' extents; every caller keeps M and N either
// multiples of the tile or equal to the remaining extent of the output.
#pragma once
#include "common.cuh"

namespace gq {

enum : int { KIND_BF16 = 0, KIND_TF32X3 = 1, KIND_BF16X3 = 2 };

// Bytes per operand element of a kind.
__host__ __device__ constexpr int kind_elem_bytes(int kind) { return kind == KIND_TF32X3 ? 4 : 2; }

struct GemmArgs {
    int M, N, K;
    int a_row0, a_col0, a_zrow, a_zcol;   // A(i,k) at map (x = a_col0 + k, y = a_row0 + i)
    int b_row0, b_col0, b_zrow, b_zcol;   // B(j,k) at map (x = b_col0 + k, y = b_row0 + j)
    int tiles_m, tiles_n;
    int batch;        // independent problems in the launch (offsets *_z* per problem)
    int triangular;   // enumerate only tiles that reach the upper triangle (nt >= tri_r * mt)
    int tri_r;        // tile M / tile N for triangular enumeration
    int k_from_m0;    // K range of a tile starts at its m0 (A upper triangular in (i,k))
    int k_to_n1;      // K range of a tile ends at n0 + tile N (B zero for k > j)
    float alpha, beta;
    float* C;
    long long ldc, c_rows, c_cols;   // extents clip the stores
    int c_row0, c_col0, c_zrow, c_zcol;
    int write_c;
    int mirror;       // also write C[j, i] for tiles above the diagonal
    int b_early;      // B was written before the grid this launch waits for began: the first
                      // tile's first stages load B before the wait (A after it)
};

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kEpiLd = 33;
constexpr int kBoxBytes = 32 * 32 * 4;           // one 32x32 fp32 box, 128-byte rows
// Tile N is a template parameter TBN (128, or 32 for launches with few tiles, whose
// epilogue stores are then spread over four times as many SMs).  Each epilogue warp owns
// a region of TBN / 32 C boxes (beta != 0) plus two boxes: the staging box and, for the
// register path of mirrored diagonal tiles, room for a padded 32x33 tile.
// Epilogue warps: eight for 128-wide tiles (two per TMEM lane quadrant, two 32-column chunks
// each), four otherwise (one per quadrant, all chunks).  Each owns three boxes: its C chunks
// (beta != 0) and a staging box for the coalesced stores.
template <int TBN>
__host__ __device__ constexpr int epi_warps() { return TBN == 128 ? 8 : 4; }
template <int TBN>
__host__ __device__ constexpr int epi_chunks_per_warp() { return (TBN / 32) / (epi_warps<TBN>() / 4); }
template <int TBN>
__host__ __device__ constexpr int epi_boxes_per_warp() { return 3; }
template <int TBN>
__host__ __device__ constexpr int epi_bytes() { return epi_warps<TBN>() * epi_boxes_per_warp<TBN>() * kBoxBytes; }   // 96 KB at TBN = 128
template <int TBN>
__host__ __device__ constexpr int gemm_threads() { return 64 + 32 * epi_warps<TBN>(); }
static_assert(epi_chunks_per_warp<128>() + 1 <= 3 && epi_chunks_per_warp<32>() + 1 <= 3, "C chunks + staging box");
static_assert(32 * kEpiLd * 4 <= 2 * kBoxBytes, "register-path staging tile fits two boxes");

template <int KIND, int TBN = BN>
struct GemmCfg {
    static_assert(TBN == 32 || TBN == 64 || TBN == 128, "tile N");
    static constexpr int KT = 128 / kind_elem_bytes(KIND);      // K elements per stage (128 bytes)
    static constexpr int NOPS = (KIND == KIND_BF16) ? 1 : 2;
    static constexpr int STAGE_BYTES = NOPS * (BM * 128 + TBN * 128);
};

template <int KIND, int STAGES, int TBN = BN>
__host__ __device__ constexpr int gemm_smem_bytes() {
    return STAGES * GemmCfg<KIND, TBN>::STAGE_BYTES + epi_bytes<TBN>() + 1024 + 256;
}

// Tiles of one problem: all of them, or (triangular) in row mt those with nt >= r * mt.
__host__ __device__ inline int tiles_of(int tiles_m, int tiles_n, int triangular, int r) {
    if (!triangular) return tiles_m * tiles_n;
    int t = 0;
    for (int mt = 0; mt < tiles_m; ++mt) t += max(0, tiles_n - r * mt);
    return t;
}

__device__ __forceinline__ void tile_coords(const GemmArgs& p, int t, int& mt, int& nt) {
    if (!p.triangular) {
        mt = t / p.tiles_n;
        nt = t % p.tiles_n;
        return;
    }
    int row = 0;
    int rem = t;
    while (row < p.tiles_m) {
        const int cnt = max(0, p.tiles_n - p.tri_r * row);
        if (rem < cnt) break;
        rem -= cnt;
        ++row;
    }
    mt = row;
    nt = p.tri_r * row + rem;
}

struct TileInfo {
    int z, mt, nt, m0, n0, kbeg, nk;
};

template <int KT, int TBN>
__device__ __forceinline__ TileInfo tile_info(const GemmArgs& p, int w, int tiles_per_batch) {
    TileInfo ti;
    ti.z = w / tiles_per_batch;
    tile_coords(p, w % tiles_per_batch, ti.mt, ti.nt);
    ti.m0 = ti.mt * BM;
    ti.n0 = ti.nt * TBN;
    ti.kbeg = p.k_from_m0 ? ti.m0 : 0;
    const int kend = p.k_to_n1 ? min(p.K, ti.n0 + TBN) : p.K;
    ti.nk = kend > ti.kbeg ? (kend - ti.kbeg + KT - 1) / KT : 0;
    return ti;
}

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

// Warp-cooperative store of a 32x32 fp32 block, given one row per lane (or, transposed,
// one column per lane), to rows y0.. and columns x0.. of a row-major matrix, clipped to
// rows x cols.  The block passes through this warp's swizzled staging box so that every
// global store instruction writes whole 128-byte row segments.  Columns come in groups of
// four (x0 and cols are multiples of 4).
__device__ __forceinline__ void emit_block(uint8_t* box, int lane, const float (&v)[32], bool transposed,
                                           float* base, long long ld, long long rows, long long cols, long long y0,
                                           long long x0) {
    __syncwarp();   // earlier readers of the box are done
    if (transposed)
        box_put_col(box, lane, v);
    else
        box_put_row(box, lane, v);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int row = 4 * i + (lane >> 3), c4 = lane & 7;
        const float4 val = *reinterpret_cast<const float4*>(box + row * 128 + ((c4 ^ (row & 7)) << 4));
        const long long gy = y0 + row, gx = x0 + 4 * c4;
        if (gy < rows && gx < cols) *reinterpret_cast<float4*>(base + gy * ld + gx) = val;
    }
}

// Error-free sum: s + e == a + b exactly (Knuth's two-sum, round-to-nearest).
__device__ __forceinline__ void two_sum(float a, float b, float& s, float& e) {
    s = __fadd_rn(a, b);
    const float bb = __fsub_rn(s, a);
    e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
}

// Chunk c (32 columns, this warp's 32 lanes) of a tile's final accumulator: the last
// segment at acc, plus (multi) the running sum of the earlier segments, plus (XACC) the
// cross-product accumulator.  Layout as in tc_gemm_kernel.
template <int TBN, bool XACC, bool TSUM>
__device__ __forceinline__ void fetch_chunk(uint32_t tmem, uint32_t acc, uint32_t lane_off, int c, bool multi,
                                            uint32_t (&r)[32]) {
    constexpr int SUM_HI = 2 * TBN, XOFF = 3 * TBN, SUM_LO = (XACC ? 4 : 3) * TBN;
    tmem_ld_32x32b_x32(acc + (uint32_t)(c * 32), r);
    float lo[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) lo[u] = 0.f;
    if (XACC) {
        uint32_t x[32];
        tmem_ld_32x32b_x32(tmem + (uint32_t)(XOFF + c * 32) + lane_off, x);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 32; ++u) lo[u] = __uint_as_float(x[u]);
    }
    if (multi) {
        uint32_t h[32];
        tmem_ld_32x32b_x32(tmem + (uint32_t)(SUM_HI + c * 32) + lane_off, h);
        if (TSUM) {
            uint32_t l[32];
            tmem_ld_32x32b_x32(tmem + (uint32_t)(SUM_LO + c * 32) + lane_off, l);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                float s, e;
                two_sum(__uint_as_float(h[u]), __uint_as_float(r[u]), s, e);
                lo[u] += __uint_as_float(l[u]) + e;
                r[u] = __float_as_uint(s);
            }
        } else {
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 32; ++u) r[u] = __float_as_uint(__uint_as_float(h[u]) + __uint_as_float(r[u]));
        }
    } else {
        tmem_ld_wait();
    }
#pragma unroll
    for (int u = 0; u < 32; ++u) r[u] = __float_as_uint(__uint_as_float(r[u]) + lo[u]);
}

template <int KIND, int STAGES, int TBN, int SEG>
__global__ void __launch_bounds__(gemm_threads<TBN>(), 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mA2,
                   const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mB2,
                   const __grid_constant__ CUtensorMap mC, const GemmArgs p) {
    using Cfg = GemmCfg<KIND, TBN>;
    constexpr int KT = Cfg::KT, NOPS = Cfg::NOPS, STAGE_BYTES = Cfg::STAGE_BYTES;
    constexpr int A_BYTES = BM * 128;
    constexpr int B_BYTES = TBN * 128;
    // Two accumulators.  Segmented accumulation adds the running sum of a tile's segments
    // and, for the tf32 kinds, an accumulator of the small cross products (hi*lo + lo*hi)
    // that spans the whole tile, so each segment accumulates only hi*hi products.
    constexpr bool XACC = SEG > 0 && KIND != KIND_BF16;
    // Where it fits, the running sum is kept as an unevaluated pair hi + lo updated by
    // two-sum, so adding the segments is exact up to the final rounding.
    constexpr bool TSUM = SEG > 0 && ((XACC ? 5 : 4) * TBN <= 512);
    constexpr int SUM_HI = 2 * TBN, SUM_LO = (XACC ? 4 : 3) * TBN;
    constexpr int TMEM_NEED = SEG > 0 ? (XACC ? 4 : 3) * TBN + (TSUM ? TBN : 0) : 2 * TBN;
    constexpr uint32_t TMEM_COLS = TMEM_NEED <= 32 ? 32u : TMEM_NEED <= 64 ? 64u : TMEM_NEED <= 128 ? 128u
                                 : TMEM_NEED <= 256 ? 256u : 512u;
    static_assert(TMEM_NEED <= 512, "tensor memory columns");


    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* epi = smem + STAGES * STAGE_BYTES;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(epi + epi_bytes<TBN>());
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* tfull_bar = empty_bar + STAGES;   // [2] accumulator ready
    uint64_t* tempty_bar = tfull_bar + 2;       // [2] accumulator drained (4 epilogue warps)
    constexpr int EPIW = epi_warps<TBN>(), CPW = epi_chunks_per_warp<TBN>();
    uint64_t* cin_bar = tempty_bar + 2;         // [EPIW] per-warp C chunk loads
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cin_bar + EPIW);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_per_batch = tiles_of(p.tiles_m, p.tiles_n, p.triangular, p.tri_r);
    const int total = tiles_per_batch * p.batch;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], EPIW);
        }
        for (int q = 0; q < EPIW; ++q) mbar_init(&cin_bar[q], 1);
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
    // b_early: the producer arms the first tile's first stages with their full byte count and
    // loads their B parts before the wait; the A parts follow it, and a stage completes only
    // when both have landed.  Every thread still signals its dependents after its own wait.
    int nearly = 0;
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&mA);
        prefetch_tmap(&mB);
        if (NOPS == 2) {
            prefetch_tmap(&mA2);
            prefetch_tmap(&mB2);
        }
        if (p.b_early && (int)blockIdx.x < total) {
            const TileInfo ti = tile_info<KT, TBN>(p, blockIdx.x, tiles_per_batch);
            const int bx = p.b_col0 + ti.z * p.b_zcol, by = p.b_row0 + ti.z * p.b_zrow + ti.n0;
            nearly = min(STAGES, ti.nk);
            for (int kt = 0; kt < nearly; ++kt) {   // fresh stages: nothing to wait for
                uint8_t* st = smem + kt * STAGE_BYTES;
                mbar_arrive_expect_tx(&full_bar[kt], STAGE_BYTES);
                const int k = ti.kbeg + kt * KT;
                tma_load_2d(st + NOPS * A_BYTES, &mB, &full_bar[kt], bx + k, by);
                if (NOPS == 2) tma_load_2d(st + NOPS * A_BYTES + B_BYTES, &mB2, &full_bar[kt], bx + k, by);
            }
        }
    }
    pdl_wait();
    pdl_trigger();

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer: one ring of stages across all tiles of this CTA
        uint32_t kiter = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
            const TileInfo ti = tile_info<KT, TBN>(p, w, tiles_per_batch);
            const int ax = p.a_col0 + ti.z * p.a_zcol, ay = p.a_row0 + ti.z * p.a_zrow + ti.m0;
            const int bx = p.b_col0 + ti.z * p.b_zcol, by = p.b_row0 + ti.z * p.b_zrow + ti.n0;
            for (int kt = 0; kt < ti.nk; ++kt, ++kiter) {
                const int s = kiter % STAGES;
                const uint32_t it = kiter / STAGES;
                uint8_t* st = smem + s * STAGE_BYTES;
                const int k = ti.kbeg + kt * KT;
                if ((int)kiter < nearly) {   // armed and its B issued before the wait
                    tma_load_2d(st, &mA, &full_bar[s], ax + k, ay);
                    if (NOPS == 2) tma_load_2d(st + A_BYTES, &mA2, &full_bar[s], ax + k, ay);
                    continue;
                }
                if (!mbar_wait(&empty_bar[s], (it & 1) ^ 1, w)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&full_bar[s], STAGE_BYTES);
                tma_load_2d(st, &mA, &full_bar[s], ax + k, ay);
                if (NOPS == 2) tma_load_2d(st + A_BYTES, &mA2, &full_bar[s], ax + k, ay);
                tma_load_2d(st + NOPS * A_BYTES, &mB, &full_bar[s], bx + k, by);
                if (NOPS == 2) tma_load_2d(st + NOPS * A_BYTES + B_BYTES, &mB2, &full_bar[s], bx + k, by);
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        constexpr uint32_t idesc = make_idesc(KIND == KIND_TF32X3 ? 2u : 1u, BM, TBN);
        uint32_t kiter = 0;
        bool ok = true;
        int seg = 0;   // accumulator segments issued by this CTA (buffer = seg & 1)
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
            const TileInfo ti = tile_info<KT, TBN>(p, w, tiles_per_batch);
            const int nkk = 4 * ti.nk;                        // MMA k-steps of the tile
            const int segk = SEG > 0 ? SEG : max(nkk, 1);     // k-steps per segment
            const uint32_t xacc = tmem + (uint32_t)(3 * TBN);
            if (XACC && seg > 0) {   // the previous tile's cross accumulator has been read
                const int pb = (seg - 1) & 1;
                if (!mbar_wait(&tempty_bar[pb], (uint32_t)((seg - 1) >> 1) & 1, w)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            // open segment: wait until its accumulator buffer has been drained
            auto open_segment = [&](uint32_t& acc_out) -> bool {
                const int buf = seg & 1;
                if (!mbar_wait(&tempty_bar[buf], (uint32_t)((seg >> 1) & 1) ^ 1u, w)) return false;
                tc_fence_after();
                acc_out = tmem + (uint32_t)(buf * TBN);
                return true;
            };
            uint32_t acc = 0;
            if (!open_segment(acc)) {
                ok = false;
                break;
            }
            int kkc = 0;      // k-steps issued in this tile
            int segpos = 0;   // k-steps issued in the open segment
            for (int kt = 0; kt < ti.nk && ok; ++kt, ++kiter) {
                const int s = kiter % STAGES;
                const uint32_t it = kiter / STAGES;
                if (!mbar_wait(&full_bar[s], it & 1, w)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t st = smem_u32(smem + s * STAGE_BYTES);
                const uint32_t a_hi = st, a_lo = st + A_BYTES;
                const uint32_t b_hi = st + NOPS * A_BYTES, b_lo = b_hi + B_BYTES;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk, ++kkc, ++segpos) {
                    if (SEG > 0 && segpos == segk) {   // close the segment, open the next
                        umma_commit(&tfull_bar[seg & 1]);
                        ++seg;
                        segpos = 0;
                        if (!open_segment(acc)) {
                            ok = false;
                            break;
                        }
                    }
                    const uint32_t off = kk * 32;
                    const uint32_t acc0 = segpos > 0 ? 1u : 0u;
                    if (KIND == KIND_BF16) {
                        umma_bf16(acc, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_hi + off), idesc, acc0);
                    } else if (KIND == KIND_BF16X3 && XACC) {
                        const uint32_t x0 = kkc > 0 ? 1u : 0u;
                        umma_bf16(acc, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_hi + off), idesc, acc0);
                        umma_bf16(xacc, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_lo + off), idesc, x0);
                        umma_bf16(xacc, desc_sw128_kmajor(a_lo + off), desc_sw128_kmajor(b_hi + off), idesc, 1u);
                    } else if (KIND == KIND_BF16X3) {
                        umma_bf16(acc, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_hi + off), idesc, acc0);
                        umma_bf16(acc, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_lo + off), idesc, 1u);
                        umma_bf16(acc, desc_sw128_kmajor(a_lo + off), desc_sw128_kmajor(b_hi + off), idesc, 1u);
                    } else if (XACC) {
                        const uint32_t x0 = kkc > 0 ? 1u : 0u;
                        umma_tf32(acc, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_hi + off), idesc, acc0);
                        umma_tf32(xacc, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_lo + off), idesc, x0);
                        umma_tf32(xacc, desc_sw128_kmajor(a_lo + off), desc_sw128_kmajor(b_hi + off), idesc, 1u);
                    } else {
                        umma_tf32(acc, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_hi + off), idesc, acc0);
                        umma_tf32(acc, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_lo + off), idesc, 1u);
                        umma_tf32(acc, desc_sw128_kmajor(a_lo + off), desc_sw128_kmajor(b_hi + off), idesc, 1u);
                    }
                }
                umma_commit(&empty_bar[s]);
            }
            if (!ok) break;
            umma_commit(&tfull_bar[seg & 1]);
            ++seg;
        }
    } else if (warp >= 2) {
        // ---------------- epilogue: warp w (2 ..) owns accumulator rows 32q .. 32q+31 of every
        // tile, q = w % 4, and the chunks c0e .. c0e + CPW - 1 of them
        const int q = warp & 3, ew = warp - 2, c0e = (ew >> 2) * CPW;
        const bool use_c = p.beta != 0.f;
        // this warp's C chunks (beta != 0), then its staging box
        uint8_t* wreg = epi + ew * epi_boxes_per_warp<TBN>() * kBoxBytes;   // this warp's region
        uint8_t* cbox = wreg;
        uint8_t* kb = wreg + CPW * kBoxBytes;                               // staging box
        float* stage_t = reinterpret_cast<float*>(wreg);   // register-path staging (own region)
        int seg = 0;
        uint32_t cin_use = 0;
        bool alive = true;
        for (int w = blockIdx.x; w < total && alive; w += gridDim.x) {
            const TileInfo ti = tile_info<KT, TBN>(p, w, tiles_per_batch);
            const int nkk = 4 * ti.nk;
            const int segk = SEG > 0 ? SEG : max(nkk, 1);
            const int nseg = max(1, (nkk + segk - 1) / segk);
            const uint32_t lane_off = (uint32_t)(q * 32) << 16;
            bool ok = true;
            // C (beta != 0) is fetched while the MMAs run
            const int zc_x = p.c_col0 + ti.z * p.c_zcol, zc_y = p.c_row0 + ti.z * p.c_zrow;
            const int iy = ti.m0 + 32 * q;
            const bool diag_mirror = p.mirror && ti.nt == ti.mt;
            const bool fetch_c = use_c && !diag_mirror;
            if (fetch_c) {
                fence_proxy_async_smem();   // this warp's reads of cbox (previous tile) come first
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_expect_tx(&cin_bar[ew], CPW * kBoxBytes);
                    for (int c = 0; c < CPW; ++c)
                        tma_load_2d(cbox + c * kBoxBytes, &mC, &cin_bar[ew], zc_x + ti.n0 + 32 * (c0e + c), zc_y + iy);
                }
                __syncwarp();
            }
            // Segments before the last: add the accumulator into the running sum (TMEM
            // columns SUM_HI .., and SUM_LO .. for two-sum) with round-to-nearest fp32
            // arithmetic, then release the buffer.
            for (int sg = 0; sg + 1 < nseg && ok; ++sg, ++seg) {
                const int sb = seg & 1;
                ok = mbar_wait(&tfull_bar[sb], (uint32_t)(seg >> 1) & 1, w);
                tc_fence_after();
#pragma unroll 1
                for (int c = c0e; c < c0e + CPW; ++c) {
                    const uint32_t src = tmem + (uint32_t)(sb * TBN + c * 32) + lane_off;
                    const uint32_t dhi = tmem + (uint32_t)(SUM_HI + c * 32) + lane_off;
                    const uint32_t dlo = tmem + (uint32_t)(SUM_LO + c * 32) + lane_off;
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(src, r);
                    if (sg > 0) {
                        uint32_t t[32];
                        tmem_ld_32x32b_x32(dhi, t);
                        if (TSUM) {
                            uint32_t e[32];
                            tmem_ld_32x32b_x32(dlo, e);
                            tmem_ld_wait();
#pragma unroll
                            for (int u = 0; u < 32; ++u) {
                                float s, er;
                                two_sum(__uint_as_float(t[u]), __uint_as_float(r[u]), s, er);
                                r[u] = __float_as_uint(s);
                                e[u] = __float_as_uint(__uint_as_float(e[u]) + er);
                            }
                            tmem_st_32x32b_x32(dlo, e);
                        } else {
                            tmem_ld_wait();
#pragma unroll
                            for (int u = 0; u < 32; ++u)
                                r[u] = __float_as_uint(__uint_as_float(r[u]) + __uint_as_float(t[u]));
                        }
                    } else {
                        tmem_ld_wait();
                        if (TSUM) {
                            uint32_t e[32];
#pragma unroll
                            for (int u = 0; u < 32; ++u) e[u] = 0u;
                            tmem_st_32x32b_x32(dlo, e);
                        }
                    }
                    tmem_st_32x32b_x32(dhi, r);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty_bar[sb]);
            }
            const int buf = seg & 1;
            const uint32_t use = (uint32_t)(seg >> 1);
            ++seg;
            ok = ok && mbar_wait(&tfull_bar[buf], use & 1, w);
            alive = ok;
            tc_fence_after();
            const uint32_t acc = tmem + (uint32_t)(buf * TBN) + lane_off;
            const bool multi = nseg > 1;   // the last segment joins a running sum
            const int n0 = ti.n0, mt = ti.mt, nt = ti.nt;
            if (!diag_mirror) {
                const bool mirror = p.mirror && nt > mt;
                const bool has_c = p.write_c != 0;
                bool cin_ok = true;
                if (fetch_c) {
                    cin_ok = mbar_wait(&cin_bar[ew], cin_use & 1, w);
                    ++cin_use;
                }
#pragma unroll 1
                for (int c = c0e; c < c0e + CPW; ++c) {
                    const int j0 = n0 + c * 32;
                    uint32_t r[32];
                    if (ti.nk > 0 && ok) {
                        fetch_chunk<TBN, XACC, TSUM>(tmem, acc, lane_off, c, multi, r);
                    } else {
#pragma unroll
                        for (int t = 0; t < 32; ++t) r[t] = 0u;
                    }
                    if (c == c0e + CPW - 1) {   // accumulator drained: the MMA warp may reuse it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tempty_bar[buf]);
                    }
                    if (j0 >= p.N) continue;
                    float out[32];
#pragma unroll
                    for (int t = 0; t < 32; ++t) out[t] = p.alpha * __uint_as_float(r[t]);
                    if (use_c && cin_ok) {
                        const uint8_t* cb = cbox + (c - c0e) * kBoxBytes;
#pragma unroll
                        for (int c4 = 0; c4 < 8; ++c4) {
                            const float4 v =
                                *reinterpret_cast<const float4*>(cb + lane * 128 + ((c4 ^ (lane & 7)) << 4));
                            out[4 * c4 + 0] = fmaf(p.beta, v.x, out[4 * c4 + 0]);
                            out[4 * c4 + 1] = fmaf(p.beta, v.y, out[4 * c4 + 1]);
                            out[4 * c4 + 2] = fmaf(p.beta, v.z, out[4 * c4 + 2]);
                            out[4 * c4 + 3] = fmaf(p.beta, v.w, out[4 * c4 + 3]);
                        }
                    }
                    if (has_c) emit_block(kb, lane, out, false, p.C, p.ldc, p.c_rows, p.c_cols, zc_y + iy, zc_x + j0);
                    if (mirror) emit_block(kb, lane, out, true, p.C, p.ldc, p.c_rows, p.c_cols, zc_y + j0, zc_x + iy);
                }
            } else {
                // Register path for diagonal tiles of mirrored outputs (C only): write j >= i
                // and its exact mirror with plain stores.
                __syncwarp();   // the staging area is this warp's own box region
                float* tile = stage_t;
                const int rbase = iy;
                const long long zr = zc_y, zcc = zc_x;
#pragma unroll 1
                for (int c = c0e; c < c0e + CPW; ++c) {
                    const int j0 = n0 + c * 32;
                    uint32_t r[32];
                    if (ti.nk > 0 && ok) {
                        fetch_chunk<TBN, XACC, TSUM>(tmem, acc, lane_off, c, multi, r);
                    } else {
#pragma unroll
                        for (int t = 0; t < 32; ++t) r[t] = 0u;
                    }
                    if (c == c0e + CPW - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tempty_bar[buf]);
                    }
                    if (j0 >= p.N) continue;
#pragma unroll
                    for (int t = 0; t < 32; ++t) tile[lane * kEpiLd + t] = __uint_as_float(r[t]);
                    __syncwarp();
                    {   // pass 1: lane = column; C read batched before use
                        const int j = j0 + lane;
                        const bool col_ok = j < p.N;
                        const int nrows = max(0, min(32, p.M - rbase));
                        float cv[32];
#pragma unroll
                        for (int rr = 0; rr < 32; ++rr)
                            cv[rr] = (p.beta != 0.f && rr < nrows && col_ok) ? p.C[(zr + rbase + rr) * p.ldc + zcc + j]
                                                                          : 0.f;
#pragma unroll
                        for (int rr = 0; rr < 32; ++rr) {
                            const int i = rbase + rr;
                            const float o = fmaf(p.beta, cv[rr], p.alpha * tile[rr * kEpiLd + lane]);
                            if (rr < nrows && col_ok && j >= i) p.C[(zr + i) * p.ldc + zcc + j] = o;
                            tile[rr * kEpiLd + lane] = o;
                        }
                    }
                    __syncwarp();
                    {   // pass 2: lane = row; exact mirror of the values just written
                        const int i = rbase + lane;
#pragma unroll 4
                        for (int t = 0; t < 32; ++t) {
                            const int jj = j0 + t;
                            if (jj < p.N && i < p.M && jj > i) p.C[(zr + jj) * p.ldc + zcc + i] = tile[lane * kEpiLd + t];
                        }
                    }
                    __syncwarp();
                }
            }
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace gq

namespace gqh {

// One operand of the GEMM: a row-major matrix [rows, cols] (K is the column index).
struct Mat {
    const void* ptr;
    uint64_t rows, cols, ld;  // elements
};

// The epilogue's output matrix C (ptr == nullptr: not written), also the matrix read when
// beta != 0 and the target of mirrored writes.
struct EpiMats {
    Mat c{nullptr, 0, 0, 0};
};

inline bool make_out_map(CUtensorMap* map, const Mat& m, const CUtensorMap& fallback, bool no_alloc = false) {
    if (!m.ptr) {
        *map = fallback;
        return true;
    }
    return no_alloc ? make_tmap_2d_uncached(map, m.ptr, 4, m.rows, m.cols, m.ld, 32, 32)
                    : make_tmap_2d(map, m.ptr, 4, m.rows, m.cols, m.ld, 32, 32);
}

// Multiprocessor count of the current device (cached per device).
int num_sms();
// A non-blocking helper stream and two timing-free events of the current device,
// created on first use and kept for the life of the process.
bool aux_stream(cudaStream_t* st, cudaEvent_t* ev0, cudaEvent_t* ev1);
// Streams of the blocked factorization, created once per device: the critical chain and
// the near updates at the highest stream priority, the far updates and the inverse at the
// lowest; events
// for the cross-stream dependencies (timing disabled).
struct FactStreams {
    cudaStream_t chain, near, far, inv;
    cudaEvent_t ev[12];
};
bool fact_streams(FactStreams* fs);

// C is read (beta != 0) only where it is also written.
inline bool epilogue_fits(const gq::GemmArgs& p) { return p.beta == 0.f || p.write_c; }

// Launch D = A B^T with the given epilogue.  For the tf32 kinds a2/b2 are the lo parts.
// max_ctas > 0 caps the persistent grid (to leave SMs to a concurrent kernel).  after_event:
// the launch follows a cross-stream event wait, so it is not a programmatic dependent.
// no_alloc: no host-side bookkeeping that allocates (tensor maps encoded afresh, the
// shared-memory attribute set directly, no per-launch timing).
template <int KIND, int STAGES, int TBN = gq::BN, int SEG = 0>
cudaError_t launch_gemm(const Mat& a, const Mat& a2, const Mat& b, const Mat& b2, const EpiMats& o, gq::GemmArgs p,
                        int batch, cudaStream_t stream, const char* name, int max_ctas = 0,
                        bool after_event = false, bool no_alloc = false) {
    using Cfg = gq::GemmCfg<KIND, TBN>;
    const int eb = gq::kind_elem_bytes(KIND);
    CUtensorMap ma, ma2, mb, mb2, mc;
    auto tmap = [no_alloc](CUtensorMap* m, const Mat& x, int elb, uint32_t br, uint32_t bc) {
        return no_alloc ? make_tmap_2d_uncached(m, x.ptr, elb, x.rows, x.cols, x.ld, br, bc)
                        : make_tmap_2d(m, x.ptr, elb, x.rows, x.cols, x.ld, br, bc);
    };
    if (p.mirror && TBN != gq::BM) return cudaErrorInvalidValue;   // mirrored outputs: square tiles only
    if (!tmap(&ma, a, eb, gq::BM, Cfg::KT)) return cudaErrorInvalidValue;
    if (!tmap(&mb, b, eb, TBN, Cfg::KT)) return cudaErrorInvalidValue;
    if (KIND != gq::KIND_BF16) {
        if (!tmap(&ma2, a2, eb, gq::BM, Cfg::KT)) return cudaErrorInvalidValue;
        if (!tmap(&mb2, b2, eb, TBN, Cfg::KT)) return cudaErrorInvalidValue;
    } else {
        ma2 = ma;
        mb2 = mb;
    }
    if (!make_out_map(&mc, o.c, ma, no_alloc)) return cudaErrorInvalidValue;
    p.C = static_cast<float*>(const_cast<void*>(o.c.ptr));
    p.ldc = (long long)o.c.ld;
    p.c_rows = (long long)o.c.rows;
    p.c_cols = (long long)o.c.cols;
    if (!epilogue_fits(p)) return cudaErrorInvalidValue;
    p.tiles_m = (p.M + gq::BM - 1) / gq::BM;
    p.tiles_n = (p.N + TBN - 1) / TBN;
    p.batch = batch;
    p.tri_r = gq::BM / TBN;
    const long long tiles = (long long)gq::tiles_of(p.tiles_m, p.tiles_n, p.triangular, p.tri_r) * batch;
    if (tiles <= 0) return cudaSuccess;
    constexpr int smem = gq::gemm_smem_bytes<KIND, STAGES, TBN>();
    auto kern = gq::tc_gemm_kernel<KIND, STAGES, TBN, SEG>;
    cudaError_t e = no_alloc ? cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)
                             : ensure_smem_attr(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)std::min<long long>(tiles, max_ctas > 0 ? max_ctas : num_sms());
    {
        TimedScope ts__(no_alloc ? nullptr : name, stream);
        constexpr int nthr = gq::gemm_threads<TBN>();
        e = after_event ? launch_plain(kern, dim3(grid), dim3(nthr), (size_t)smem, stream, ma, ma2, mb, mb2, mc, p)
                        : launch_pdl(kern, dim3(grid), dim3(nthr), (size_t)smem, stream, ma, ma2, mb, mb2, mc, p);
    }
    return e != cudaSuccess ? e : cudaGetLastError();
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
