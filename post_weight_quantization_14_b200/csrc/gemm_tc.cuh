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
// 2..5 read the accumulator from tensor memory and run the epilogue.  Every wait is
// bounded (GPTQ_ERR_TIMEOUT).  No TMA multicast.
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
    float* T_hi;
    float* T_lo;
    long long ldt;
    int t_row0, t_col0, t_zrow, t_zcol;
};

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

template <int KIND, int BN, int STAGES>
__global__ void __launch_bounds__(192, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mA2,
                   const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mB2,
                   const GemmArgs p) {
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
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* acc_bar = empty_bar + STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_bar + 1);

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
        const int q = warp & 3;
        const int i = m0 + q * 32 + lane;
        const bool row_ok = i < p.M;
        const bool mirror = p.mirror && nt > mt;
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
            const int jn = min(32, p.N - j0);
            float out[32];
            if (row_ok) {
                const long long ar = p.c_row0 + z * p.c_zrow + i;
                const long long ac = p.c_col0 + z * p.c_zcol + j0;
                const long long crow = ar * p.ldc + ac;
                int jc = jn;
                if (p.c_lim_rows > 0 && ar >= p.c_lim_rows) jc = 0;
                if (p.c_lim_cols > 0) jc = (int)max(0LL, min((long long)jc, (long long)p.c_lim_cols - ac));
                const bool vec = (jc == 32) && ((crow & 3) == 0);
                if (p.beta != 0.f) {
                    if (vec) {
                        const float4* src = reinterpret_cast<const float4*>(p.C + crow);
#pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            float4 cv = src[t];
                            out[4 * t + 0] = p.alpha * __uint_as_float(r[4 * t + 0]) + p.beta * cv.x;
                            out[4 * t + 1] = p.alpha * __uint_as_float(r[4 * t + 1]) + p.beta * cv.y;
                            out[4 * t + 2] = p.alpha * __uint_as_float(r[4 * t + 2]) + p.beta * cv.z;
                            out[4 * t + 3] = p.alpha * __uint_as_float(r[4 * t + 3]) + p.beta * cv.w;
                        }
                    } else {
#pragma unroll
                        for (int t = 0; t < 32; ++t)
                            out[t] = p.alpha * __uint_as_float(r[t]) +
                                     (t < jc ? p.beta * p.C[crow + t] : 0.f);
                    }
                } else {
#pragma unroll
                    for (int t = 0; t < 32; ++t) out[t] = p.alpha * __uint_as_float(r[t]);
                }
                if (p.write_c) {
                    if (vec) {
                        float4* dst = reinterpret_cast<float4*>(p.C + crow);
#pragma unroll
                        for (int t = 0; t < 8; ++t)
                            dst[t] = make_float4(out[4 * t], out[4 * t + 1], out[4 * t + 2], out[4 * t + 3]);
                    } else {
#pragma unroll
                        for (int t = 0; t < 32; ++t)
                            if (t < jc) p.C[crow + t] = out[t];
                    }
                }
                if (p.S_hi) {
                    const long long srow = (long long)(p.s_row0 + z * p.s_zrow + i) * p.lds +
                                           (p.s_col0 + z * p.s_zcol + j0);
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        if (t < jn) store_split(p.S_hi, p.S_lo, srow + t, out[t]);
                }
            }
            // transposed outputs: for fixed t the warp writes 32 consecutive rows i -> coalesced
            if (p.T_hi) {
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    if (t < jn && row_ok) {
                        const long long idx = (long long)(p.t_row0 + z * p.t_zrow + j0 + t) * p.ldt +
                                              (p.t_col0 + z * p.t_zcol + i);
                        store_split(p.T_hi, p.T_lo, idx, out[t]);
                    }
                }
            }
            if (mirror) {
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    if (t < jn && row_ok) {
                        const long long idx = (long long)(p.c_row0 + z * p.c_zrow + j0 + t) * p.ldc +
                                              (p.c_col0 + z * p.c_zcol + i);
                        p.C[idx] = out[t];
                    }
                }
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

template <int KIND, int BN, int STAGES>
constexpr int gemm_smem_bytes() {
    return STAGES * GemmCfg<KIND>::NOPS * (128 * 128 + BN * 128) + 1024 + 256;
}

}  // namespace gq

namespace gqh {

// One operand of the GEMM: a row-major matrix [rows, cols] (K is the column index).
struct Mat {
    const void* ptr;
    uint64_t rows, cols, ld;  // elements
};

// Launch D = A B^T with the given epilogue.  For KIND_TF32X3 a2/b2 are the lo parts.
template <int KIND, int BN, int STAGES>
cudaError_t launch_gemm(const Mat& a, const Mat& a2, const Mat& b, const Mat& b2, gq::GemmArgs p,
                        int batch, cudaStream_t stream, const char* name) {
    using Cfg = gq::GemmCfg<KIND>;
    const int eb = (KIND == gq::KIND_BF16) ? 2 : 4;
    CUtensorMap ma, ma2, mb, mb2;
    if (!make_tmap_2d(&ma, a.ptr, eb, a.rows, a.cols, a.ld, 128, Cfg::KT)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&mb, b.ptr, eb, b.rows, b.cols, b.ld, BN, Cfg::KT)) return cudaErrorInvalidValue;
    if (KIND == gq::KIND_TF32X3) {
        if (!make_tmap_2d(&ma2, a2.ptr, eb, a2.rows, a2.cols, a2.ld, 128, Cfg::KT))
            return cudaErrorInvalidValue;
        if (!make_tmap_2d(&mb2, b2.ptr, eb, b2.rows, b2.cols, b2.ld, BN, Cfg::KT))
            return cudaErrorInvalidValue;
    } else {
        ma2 = ma;
        mb2 = mb;
    }
    p.tiles_m = (p.M + 127) / 128;
    p.tiles_n = (p.N + BN - 1) / BN;
    long long tiles = p.triangular ? (long long)p.tiles_m * (p.tiles_m + 1) / 2
                                   : (long long)p.tiles_m * p.tiles_n;
    if (tiles <= 0 || batch <= 0) return cudaSuccess;
    constexpr int smem = gq::gemm_smem_bytes<KIND, BN, STAGES>();
    auto kern = gq::tc_gemm_kernel<KIND, BN, STAGES>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)tiles, 1, (unsigned)batch);
    {
        TimedScope ts__(name, stream);
        kern<<<grid, 192, smem, stream>>>(ma, ma2, mb, mb2, p);
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
