// Dequantizing GEMM on the packed GPTQ format, the consumer of the column loop's output:
//
//   Y[m, n] = sum_k X[m, k] W_hat[n, k],   W_hat[n, k] = s[g(k), n] (q[n, k] - z[g(k), n])
//
// (GPTQ tutorial page, "阶段三：量化与反量化": a weight is its integer times its scale;
// group-size article: one scale and zero per group of consecutive weights along the input
// dimension; the inference-kernel notes on the pages: when group boundaries coincide
// with the tile's K boundaries a group's scales are loaded once per tile.)
//
// Arithmetic.  q - z is a small integer, exact in bf16, so each group's partial product
// P_g = X (q - z)^T is formed on the tensor cores from exact products with fp32
// accumulation over the group's K range; the epilogue adds s_g * P_g into fp32 running
// sums.  The scale is applied once per group and output, as in the definition, and no
// rounded copy of W_hat is ever formed.
//
// Persistent kernel, one CTA per SM over 128 x 128 output tiles, 576 threads:
//   warp 0       TMA: the X tile (128 rows x 64 bf16, 128-byte swizzle) and the packed
//                words of the weight tile (KWT words x 128 rows, no swizzle) into a ring
//                of stages;
//   warp 1       MMA issuer (kind::f16, bf16, M = N = 128, four K = 16 steps per stage);
//                one accumulator segment per quantization group, two TMEM buffers;
//   warps 2-9    converters: two threads per weight row n0 + t, each unpacking half of
//                the row's 64 weights into bf16 (q - z), written as row t of the stage's
//                B tile in the 128-byte-swizzled K-major layout (the layout TMA would
//                produce), then fenced for the async proxy;
//   warps 10-17  epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 and one half of
//                the tile's columns, scales each segment by its group's fp16 scales and
//                adds it into fp32 running sums kept in TMEM, and after the tile's last
//                segment writes Y through swizzled staging boxes with 16-byte stores.
// 576 threads: each of the SM's four partitions holds up to five warps, so the launch
// bound caps the registers at 96 per thread (the epilogue keeps its sums in TMEM).
// Every wait is bounded (GPTQ_ERR_TIMEOUT).  No TMA multicast.
#pragma once
#include <cuda_bf16.h>

#include "gemm_tc.cuh"
#include "pack.cuh"

namespace gq {

constexpr int DQ_BM = 128, DQ_BN = 128, DQ_BK = 64;
constexpr int DQ_THREADS = 576;
constexpr int DQ_CONV_WARP0 = 2, DQ_EPI_WARP0 = 10;   // eight converter warps, eight epilogue warps

template <int BITS>
struct DqCfg {
    static constexpr int KWT = DQ_BK * BITS / 32;   // packed words per weight row and k-tile
    static constexpr int A_BYTES = DQ_BM * 128;     // 128 rows of 64 bf16
    static constexpr int B_BYTES = DQ_BN * 128;
    static constexpr int P_BYTES = KWT * DQ_BN * 4;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + P_BYTES;
    static constexpr int STAGES = BITS == 8 ? 3 : 4;   // within 227 KB of shared memory
    static_assert(STAGE_BYTES % 1024 == 0, "each stage's tiles stay 1024-byte aligned");
};

template <int BITS>
__host__ __device__ constexpr int dq_smem_bytes() {
    return 1024 + DqCfg<BITS>::STAGES * DqCfg<BITS>::STAGE_BYTES + 16 * kBoxBytes + 8 * 256 + 256;
}

struct DqArgs {
    const __half* scales;    // [n_groups, N]
    const int32_t* qzeros;   // [n_groups, ceil(N * BITS / 32)], or null when symmetric
    float* Y;                // [M, N] row-major
    int M, N, K;
    int kpg;                 // k-tiles per quantization group
    int tiles_m, tiles_n;
};

// Eight consecutive weights k = 8c .. 8c+7 of one row as bf16 (q - z), from that row's
// packed words col[j * DQ_BN].  zz holds (128 + z) twice for the 2- and 4-bit forms.
template <int BITS>
__device__ __forceinline__ uint4 dq_chunk(const uint32_t* col, int c, int z, __nv_bfloat162 zz) {
    uint32_t out[4];
    if constexpr (BITS == 8) {
        const uint32_t w0 = col[(2 * c) * DQ_BN], w1 = col[(2 * c + 1) * DQ_BN];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int a0 = (int)((w0 >> (16 * i)) & 0xFFu) - z, a1 = (int)((w0 >> (16 * i + 8)) & 0xFFu) - z;
            const int b0 = (int)((w1 >> (16 * i)) & 0xFFu) - z, b1 = (int)((w1 >> (16 * i + 8)) & 0xFFu) - z;
            const __nv_bfloat162 pa = __floats2bfloat162_rn((float)a0, (float)a1);   // |q - z| <= 255: exact
            const __nv_bfloat162 pb = __floats2bfloat162_rn((float)b0, (float)b1);
            out[i] = *reinterpret_cast<const uint32_t*>(&pa);
            out[2 + i] = *reinterpret_cast<const uint32_t*>(&pb);
        }
    } else if constexpr (BITS == 4) {
        // 0x4300 | q is the bf16 of 128 + q (q < 128); subtracting 128 + z is exact.  Byte
        // permutes put the even and odd nibbles of the word side by side in 16-bit lanes.
        const uint32_t w = col[c * DQ_BN];
        const uint32_t even = w & 0x0F0F0F0Fu, odd = (w >> 4) & 0x0F0F0F0Fu;
        const uint32_t q03 = __byte_perm(even, odd, 0x5140), q47 = __byte_perm(even, odd, 0x7362);
        const uint32_t v[4] = {__byte_perm(q03, 0x43434343u, 0x4140), __byte_perm(q03, 0x43434343u, 0x4342),
                               __byte_perm(q47, 0x43434343u, 0x4140), __byte_perm(q47, 0x43434343u, 0x4342)};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 d = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&v[i]), zz);
            out[i] = *reinterpret_cast<const uint32_t*>(&d);
        }
    } else {
        // 0x4300 | q is the bf16 of 128 + q (q < 128); subtracting 128 + z is exact.
        const uint32_t w = col[(c >> 1) * DQ_BN] >> ((c & 1) * 16);
        constexpr uint32_t M = (1u << BITS) - 1u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = (w >> (2 * BITS * i)) & M, hi = (w >> (2 * BITS * i + BITS)) & M;
            const uint32_t v = lo | (hi << 16) | 0x43004300u;
            const __nv_bfloat162 d = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&v), zz);
            out[i] = *reinterpret_cast<const uint32_t*>(&d);
        }
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

template <int BITS>
__global__ void __launch_bounds__(DQ_THREADS, 1)
    dq_gemm_kernel(const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mP, const DqArgs p) {
    using Cfg = DqCfg<BITS>;
    constexpr int A_BYTES = Cfg::A_BYTES, B_BYTES = Cfg::B_BYTES, STAGE_BYTES = Cfg::STAGE_BYTES;
    constexpr int STAGES = Cfg::STAGES;
    constexpr uint32_t SUM_COL = 2 * DQ_BN;    // running sums after the two segment buffers
    constexpr uint32_t TMEM_COLS = 512;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* epi = smem + STAGES * STAGE_BYTES;
    uint8_t* scale_buf = epi + 16 * kBoxBytes;                                 // [8 warps][2][64] fp16
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(scale_buf + 8 * 256);    // TMA landed
    uint64_t* conv_bar = full_bar + STAGES;                                 // B tile written
    uint64_t* empty_bar = conv_bar + STAGES;                                // MMAs done
    uint64_t* tfull_bar = empty_bar + STAGES;                               // [2] segment ready
    uint64_t* tempty_bar = tfull_bar + 2;                                      // [2] segment drained
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty_bar + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total = p.tiles_m * p.tiles_n;
    const int nkt = p.K / DQ_BK;
    const int nseg = nkt / p.kpg;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&conv_bar[s], 8);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], 8);
        }
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
    pdl_wait();

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer
        prefetch_tmap(&mX);
        prefetch_tmap(&mP);
        uint32_t kiter = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
            const int m0 = (w % p.tiles_m) * DQ_BM, n0 = (w / p.tiles_m) * DQ_BN;
            for (int kt = 0; kt < nkt; ++kt, ++kiter) {
                const int s = kiter % STAGES;
                const uint32_t it = kiter / STAGES;
                if (!mbar_wait(&empty_bar[s], (it & 1) ^ 1, w)) {
                    ok = false;
                    break;
                }
                uint8_t* st = smem + s * STAGE_BYTES;
                mbar_arrive_expect_tx(&full_bar[s], A_BYTES + Cfg::P_BYTES);
                tma_load_2d(st, &mX, &full_bar[s], kt * DQ_BK, m0);
                tma_load_2d(st + A_BYTES + B_BYTES, &mP, &full_bar[s], n0, kt * Cfg::KWT);
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        constexpr uint32_t idesc = make_idesc(1u, DQ_BM, DQ_BN);
        uint32_t kiter = 0;
        int seg = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
            for (int sg = 0; sg < nseg && ok; ++sg) {
                const int buf = seg & 1;
                if (!mbar_wait(&tempty_bar[buf], (uint32_t)((seg >> 1) & 1) ^ 1u, w)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(buf * DQ_BN);
                for (int kt = 0; kt < p.kpg; ++kt, ++kiter) {
                    const int s = kiter % STAGES;
                    const uint32_t it = kiter / STAGES;
                    if (!mbar_wait(&full_bar[s], it & 1, w) || !mbar_wait(&conv_bar[s], it & 1, w)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a = smem_u32(smem + s * STAGE_BYTES), b = a + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(acc, desc_sw128_kmajor(a + kk * 32), desc_sw128_kmajor(b + kk * 32), idesc,
                                  (kt > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty_bar[s]);
                }
                if (!ok) break;
                umma_commit(&tfull_bar[buf]);
                ++seg;
            }
        }
    } else if (warp >= DQ_CONV_WARP0 && warp < DQ_EPI_WARP0) {
        // ---------------- converters: thread tc owns half (four 16-byte chunks) of row t
        const int tc = threadIdx.x - 32 * DQ_CONV_WARP0;
        const int t = tc & (DQ_BN - 1), c0 = 4 * (tc >> 7);
        const long long zwords = ((long long)p.N * BITS + 31) / 32;
        uint32_t kiter = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
            const int n = (w / p.tiles_m) * DQ_BN + t;
            int z = 1 << (BITS - 1);
            __nv_bfloat162 zz = __floats2bfloat162_rn(0.f, 0.f);
            for (int kt = 0; kt < nkt; ++kt, ++kiter) {
                const int s = kiter % STAGES;
                const uint32_t it = kiter / STAGES;
                if (kt % p.kpg == 0) {   // a new group: this row's zero point
                    if (p.qzeros != nullptr)
                        z = n < p.N ? (int)stream_code(p.qzeros + (long long)(kt / p.kpg) * zwords, 1, n, BITS) : 0;
                    zz = __floats2bfloat162_rn(128.f + (float)z, 128.f + (float)z);
                }
                if (!mbar_wait(&full_bar[s], it & 1, w)) {
                    ok = false;
                    break;
                }
                uint8_t* st = smem + s * STAGE_BYTES;
                const uint32_t* col = reinterpret_cast<const uint32_t*>(st + A_BYTES + B_BYTES) + t;
                uint8_t* row = st + A_BYTES + (t >> 3) * 1024 + (t & 7) * 128;
#pragma unroll
                for (int c = c0; c < c0 + 4; ++c)
                    *reinterpret_cast<uint4*>(row + ((c ^ (t & 7)) << 4)) = dq_chunk<BITS>(col, c, z, zz);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&conv_bar[s]);
            }
        }
    } else if (warp >= DQ_EPI_WARP0) {
        // ---------------- epilogue
        const int ew = warp - DQ_EPI_WARP0;
        const int qd = warp & 3;               // TMEM lanes 32 qd .. 32 qd + 31
        const int h = ew >> 2;                 // columns 64 h .. 64 h + 63 of the tile
        const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
        uint8_t* box = epi + 2 * ew * kBoxBytes;   // two staging boxes per warp
        int seg = 0;
        bool alive = true;
        for (int w = blockIdx.x; w < total && alive; w += gridDim.x) {
            const int m0 = (w % p.tiles_m) * DQ_BM, n0 = (w / p.tiles_m) * DQ_BN;
            const int nc = n0 + 64 * h;        // first column of this warp
            // This warp's 64 scales of a group are fetched into shared memory one segment
            // ahead (cp.async, eight lanes x 16 bytes), so their L2 latency overlaps the
            // wait for the segment's accumulator.
            uint8_t* sbuf = scale_buf + ew * 256;
            auto prefetch_scales = [&](int sg, int slot) {
                if (lane < 8) {
                    const int n = nc + 8 * lane;
                    const __half* src = p.scales + (long long)sg * p.N + (n < p.N ? n : 0);
                    const uint32_t bytes = n < p.N ? 16u : 0u;   // zero fill past N
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                                     smem_u32(sbuf + slot * 128 + 16 * lane)),
                                 "l"(src), "r"(bytes)
                                 : "memory");
                }
                asm volatile("cp.async.commit_group;" ::: "memory");
            };
            prefetch_scales(0, 0);
            for (int sg = 0; sg < nseg; ++sg, ++seg) {
                const int buf = seg & 1;
                if (sg + 1 < nseg) {
                    prefetch_scales(sg + 1, (sg + 1) & 1);
                    asm volatile("cp.async.wait_group 1;" ::: "memory");
                } else {
                    asm volatile("cp.async.wait_group 0;" ::: "memory");
                }
                __syncwarp();
                const bool ok = mbar_wait(&tfull_bar[buf], (uint32_t)(seg >> 1) & 1, w);
                tc_fence_after();
                if (ok) {
                    const uint8_t* srow = sbuf + (sg & 1) * 128;   // this group's 64 scales
                    const bool last = sg + 1 == nseg;
#pragma unroll 1
                    for (int c = 0; c < 2; ++c) {
                        const uint32_t col = (uint32_t)(64 * h + 32 * c);
                        uint32_t r[32], t[32];
                        tmem_ld_32x32b_x32(tmem + (uint32_t)(buf * DQ_BN) + col + lane_off, r);
                        if (sg > 0) tmem_ld_32x32b_x32(tmem + SUM_COL + col + lane_off, t);
                        tmem_ld_wait();
#pragma unroll
                        for (int j8 = 0; j8 < 4; ++j8) {
                            const uint4 sv = *reinterpret_cast<const uint4*>(srow + 64 * c + 16 * j8);
                            const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&sw[u]));
                                const int j = 8 * j8 + 2 * u;
                                const float a0 = sg > 0 ? __uint_as_float(t[j]) : 0.f;
                                const float a1 = sg > 0 ? __uint_as_float(t[j + 1]) : 0.f;
                                r[j] = __float_as_uint(fmaf(f.x, __uint_as_float(r[j]), a0));
                                r[j + 1] = __float_as_uint(fmaf(f.y, __uint_as_float(r[j + 1]), a1));
                            }
                        }
                        if (last) {   // final values straight into this chunk's staging box
                            uint8_t* b = box + c * kBoxBytes;
#pragma unroll
                            for (int c4 = 0; c4 < 8; ++c4)
                                *reinterpret_cast<uint4*>(b + lane * 128 + ((c4 ^ (lane & 7)) << 4)) =
                                    make_uint4(r[4 * c4], r[4 * c4 + 1], r[4 * c4 + 2], r[4 * c4 + 3]);
                        } else {
                            tmem_st_32x32b_x32(tmem + SUM_COL + col + lane_off, r);
                        }
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty_bar[buf]);
                if (!ok) {
                    alive = false;
                    break;
                }
            }
            if (!alive) break;
            // coalesced 16-byte stores of the two staged 32x32 blocks, clipped to M x N
            __syncwarp();
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int row = 4 * i + (lane >> 3), c4 = lane & 7;
                    const float4 val =
                        *reinterpret_cast<const float4*>(box + c * kBoxBytes + row * 128 + ((c4 ^ (row & 7)) << 4));
                    const long long gy = m0 + 32 * qd + row, gx = nc + 32 * c + 4 * c4;
                    if (gy < p.M && gx < p.N) *reinterpret_cast<float4*>(p.Y + gy * p.N + gx) = val;
                }
            }
            __syncwarp();   // the boxes are rewritten by the next tile's last segment
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

// Y = X W_hat^T for bits 2, 4, 8; K % 64 == 0, group size a multiple of 64 dividing K
// (or one group per row), N % 8 == 0.  X bf16 [M, K], 16-byte aligned.
template <int BITS>
cudaError_t dq_gemm_run(const void* X, long long M, const int32_t* qweight, const __half* scales,
                        const int32_t* qzeros, long long N, long long K, int g, float* Y, cudaStream_t st) {
    CUtensorMap mx, mp;
    if (!make_tmap_2d(&mx, X, 2, (uint64_t)M, (uint64_t)K, (uint64_t)K, gq::DQ_BM, gq::DQ_BK))
        return cudaErrorInvalidValue;
    if (!make_tmap_2d_plain(&mp, qweight, (uint64_t)(K * BITS / 32), (uint64_t)N, (uint64_t)N,
                            gq::DqCfg<BITS>::KWT, gq::DQ_BN))
        return cudaErrorInvalidValue;
    gq::DqArgs p;
    p.scales = scales;
    p.qzeros = qzeros;
    p.Y = Y;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.kpg = (int)((g < 0 ? K : g) / gq::DQ_BK);
    p.tiles_m = (int)((M + gq::DQ_BM - 1) / gq::DQ_BM);
    p.tiles_n = (int)((N + gq::DQ_BN - 1) / gq::DQ_BN);
    const long long tiles = (long long)p.tiles_m * p.tiles_n;
    constexpr int smem = gq::dq_smem_bytes<BITS>();
    auto kern = gq::dq_gemm_kernel<BITS>;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)std::min<long long>(tiles, num_sms());
    {
        TimedScope ts__("dq_gemm", st);
        e = launch_plain(kern, dim3(grid), dim3(gq::DQ_THREADS), (size_t)smem, st, mx, mp, p);
    }
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace gqh
