// GPTQ column loop of one 128-column lazy block on the tensor cores (tutorial "阶段二":
// greedy column order, errors pushed into the not-yet-quantized columns; "阶段三" and the
// group-size article: group-wise scale and zero from the current values).
//
// One CTA owns 128 rows, one thread per row (the row's tensor-memory lane).  The block
// is walked in eight sub-blocks of 16 columns.  A row's current value of a column of
// sub-block t is
//   W (global)  +  the errors of sub-blocks <= t-2 pushed by the tensor cores (in tensor
//   memory)  +  the errors of sub-block t-1 and of t's earlier columns pushed in registers,
// so that the tensor-core product of sub-block t runs while sub-block t+1 is rounded:
//   * the 16 rounding steps of sub-block t run in registers; each error d_c is pushed with
//     the normalised rows of U (d_c U[c, c'] / U[c, c]) into t's later columns and into
//     all 16 columns of sub-block t+1;
//   * the errors e_c = d_c / U_cc of sub-block t, negated and split into two tf32 parts,
//     form the A operand of three tcgen05 MMAs (hi*hi, hi*lo, lo*hi; K = 16) against the
//     block's U^T tile, which add -sum_c e_c U[c, n] to the columns n of sub-blocks >= t+2
//     (the MMA's N range starts there, so it never touches columns being read);
//   * at a group's first column the group's scale and zero come from its current values.
// The U^T tile (128 KB, both tf32 parts) arrives by TMA with 128-byte swizzle; the errors
// go to shared memory in the same K-major swizzled layout (two buffers: sub-block t+1
// writes one while the product of t reads the other).  The codes are packed into the
// output bit stream as they are formed; at the end the kernel writes the per-row sum of
// e^2, and throughout the errors as a bf16 split (operand of the trailing update).  Every
// wait is bounded.
#pragma once
#include "colloop.cuh"

namespace gq {

constexpr int TC_SUB = 16;                 // sub-block width
constexpr int TC_NSUB = CB / TC_SUB;       // sub-blocks per block
constexpr int TC_ROWS = 128;               // rows per CTA (tensor-memory lanes)
constexpr int TC_UNW = 2 * TC_SUB;         // normalised U entries per row: own sub-block + next
constexpr int TC_UN = TC_NSUB * TC_SUB * TC_UNW;   // floats of the normalised U rows of a block

// shared-memory layout (offsets from a 1024-aligned base)
constexpr uint32_t TCS_BH = 0;                       // U^T tile hi: 4 boxes [128 n][32 k] fp32
constexpr uint32_t TCS_BL = TCS_BH + 65536;          // U^T tile lo
constexpr uint32_t TCS_A = TCS_BL + 65536;           // -E: 2 buffers x {hi, lo} x [128 rows][32 k] (k < 16 used)
constexpr uint32_t TCS_UN = TCS_A + 4 * 16384;       // [8][16][32] normalised U rows
constexpr uint32_t TCS_INVD = TCS_UN + TC_UN * 4;    // [128] 1 / U_cc
constexpr uint32_t TCS_BARS = TCS_INVD + 512;
constexpr uint32_t TCS_BYTES = TCS_BARS + 64;
constexpr int TC_SMEM = (int)TCS_BYTES + 1024;        // + alignment slack
static_assert(TCS_BARS % 8 == 0, "barrier alignment");
static_assert(TC_SMEM <= 227 * 1024, "shared memory");

struct TcColArgs {
    const float* W;
    long long d_out, d_in;
    int c0, nc, blk;
    const float* un;        // this block's normalised U rows [8][16][32]
    const float* inv_d;     // [d_in] 1 / U_cc
    int g, sym;
    const float* row_scale;
    const float* row_zero;
    int32_t* qweight;
    __half* scales;
    uint8_t* zeros_u8;
    uint16_t* E_hi;         // errors of this block: E[row * e_ld + e_col0 + col], bf16 split
    uint16_t* E_lo;
    long long e_ld;
    int e_col0;
    float* err_sq;
    int first_block;
};

__device__ __forceinline__ uint32_t sw128_off(int row, int k) {   // fp32 element (row, k) of a K-major SW128 tile
    return (uint32_t)(row * 128 + ((((k >> 2) ^ (row & 7))) << 4) + (k & 3) * 4);
}

template <int BITS>
__global__ void __launch_bounds__(TC_ROWS, 1)
    colloop_tc_kernel(const __grid_constant__ CUtensorMap mBh, const __grid_constant__ CUtensorMap mBl,
                      const TcColArgs p) {
    extern __shared__ uint8_t tc_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_raw) + 1023) & ~uintptr_t(1023));
    const float* un = reinterpret_cast<const float*>(sm + TCS_UN);
    float* invd = reinterpret_cast<float*>(sm + TCS_INVD);
    uint64_t* bar_b = reinterpret_cast<uint64_t*>(sm + TCS_BARS);
    uint64_t* bar_mma = bar_b + 1;   // [2]: the product of sub-block t commits to bar_mma[t & 1]
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bar_b + 3);
    constexpr int MAXQ = (1 << BITS) - 1;
    constexpr unsigned FULL = 0xffffffffu;
    const int tid = threadIdx.x, warp = tid >> 5;
    const long long row = (long long)blockIdx.x * TC_ROWS + tid;
    const bool row_ok = row < p.d_out;
    const int nsub = (p.nc + TC_SUB - 1) / TC_SUB;
    const long long where = -1 - (long long)blockIdx.x;

    if (tid == 0) {
        mbar_init(bar_b, 1);
        mbar_init(&bar_mma[0], 1);
        mbar_init(&bar_mma[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;                          // columns 0..127: hi*hi; 128..255: cross products
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    // the U-derived operands were prepared before the column loop started: they load while
    // the previous kernel (the update of this block by the previous one) finishes
    if (tid == 0) {
        prefetch_tmap(&mBh);
        prefetch_tmap(&mBl);
        mbar_arrive_expect_tx(bar_b, 2 * 65536);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            tma_load_2d(sm + TCS_BH + q * 16384, &mBh, bar_b, 32 * q, p.blk * TC_ROWS);
            tma_load_2d(sm + TCS_BL + q * 16384, &mBl, bar_b, 32 * q, p.blk * TC_ROWS);
        }
    }
    {
        const float4* src = reinterpret_cast<const float4*>(p.un);
        float4* dst = reinterpret_cast<float4*>(sm + TCS_UN);
        for (int e = tid; e < TC_UN / 4; e += TC_ROWS) dst[e] = src[e];
    }
    invd[tid] = (tid < p.nc) ? p.inv_d[p.c0 + tid] : 0.f;
    pdl_wait();   // W is written by the previous kernel
    pdl_trigger();

    const float* wrow = p.W + row * p.d_in + p.c0;
    auto load_sub = [&](int s, float (&v)[TC_SUB]) {
#pragma unroll
        for (int c = 0; c < TC_SUB; c += 4) {
            const int col = TC_SUB * s + c;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (row_ok && col < p.nc) x = *reinterpret_cast<const float4*>(wrow + col);   // nc % 8 == 0
            v[c] = x.x;
            v[c + 1] = x.y;
            v[c + 2] = x.z;
            v[c + 3] = x.w;
        }
    };
    // the product of sub-block t has committed (it may be waited for more than once)
    auto wait_mma = [&](int t) -> bool {
        if (t < 0 || t + 2 >= TC_NSUB || TC_SUB * (t + 2) >= p.nc) return true;   // never issued
        const bool r = mbar_wait(&bar_mma[t & 1], (uint32_t)((t >> 1) & 1), where);
        tc_fence_after();
        return r;
    };
    QuadState st{1.f, 1.f, 0.f, (float)MAXQ};
    if (p.g < 0 && row_ok) {
        const float z = p.row_zero[row];
        st.s = p.row_scale[row];
        st.inv_s = __frcp_rn(st.s);
        st.qlo = -z;
        st.qhi = (float)MAXQ - z;
    }
    float wcur[TC_SUB];   // sub-block t: W + pushed errors of t-1 (registers); + tensor memory below
    load_sub(0, wcur);
    bool ok = mbar_wait(bar_b, 0, where);
    __syncthreads();   // un, invd visible
    float esum = 0.f;
    bool finite = true;
    unsigned long long bits_acc = 0;   // code bit stream of the row, flushed in 32-bit words
    int nbits = 0;
    long long word = (long long)p.c0 * BITS / 32;                     // c0 * BITS is a multiple of 32
    const long long wend = ((long long)(p.c0 + p.nc) * BITS + 31) / 32;   // words of the row up to this block's end
    for (int t = 0; t < nsub && ok; ++t) {
        const int cb = TC_SUB * t;
        float wnext[TC_SUB];   // sub-block t+1: W now, its pushed errors from t added below
        if (t + 1 < nsub) load_sub(t + 1, wnext);
        float w[TC_SUB];
#pragma unroll
        for (int c = 0; c < TC_SUB; ++c) w[c] = wcur[c];
        if (t >= 2) {   // the products of sub-blocks <= t-2
            ok = wait_mma(t - 2);
            if (!ok) break;
            uint32_t a[TC_SUB], x[TC_SUB];
            tmem_ld_32x32b_x16(lane_base + (uint32_t)cb, a);
            tmem_ld_32x32b_x16(lane_base + (uint32_t)(CB + cb), x);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < TC_SUB; ++c) w[c] += __uint_as_float(a[c]) + __uint_as_float(x[c]);
        }
        // group parameters at the group's first column, from the group's current values
        if (p.g > 0 && (cb & (p.g - 1)) == 0) {
            float mn = INFINITY, mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < TC_SUB; ++c)
                if (cb + c < p.nc) {
                    mn = fminf(mn, w[c]);
                    mx = fmaxf(mx, w[c]);
                }
            if (p.g > TC_SUB && t > 0) ok = ok && wait_mma(t - 1);   // its columns past sub-block t
            for (int u = 1; u < p.g / TC_SUB && t + u < nsub; u += 2) {   // two sub-blocks per round trip
                const bool two = u + 1 < p.g / TC_SUB && t + u + 1 < nsub;
                float v[TC_SUB], v2[TC_SUB];
                load_sub(t + u, v);
                if (two) load_sub(t + u + 1, v2);
                if (t > 0) {
                    uint32_t a[TC_SUB], x[TC_SUB];
                    tmem_ld_32x32b_x16(lane_base + (uint32_t)(cb + TC_SUB * u), a);
                    tmem_ld_32x32b_x16(lane_base + (uint32_t)(CB + cb + TC_SUB * u), x);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < TC_SUB; ++c) v[c] += __uint_as_float(a[c]) + __uint_as_float(x[c]);
                    if (two) {
                        tmem_ld_32x32b_x16(lane_base + (uint32_t)(cb + TC_SUB * (u + 1)), a);
                        tmem_ld_32x32b_x16(lane_base + (uint32_t)(CB + cb + TC_SUB * (u + 1)), x);
                        tmem_ld_wait();
#pragma unroll
                        for (int c = 0; c < TC_SUB; ++c) v2[c] += __uint_as_float(a[c]) + __uint_as_float(x[c]);
                    }
                }
#pragma unroll
                for (int c = 0; c < TC_SUB; ++c) {
                    if (cb + TC_SUB * u + c < p.nc) {
                        mn = fminf(mn, v[c]);
                        mx = fmaxf(mx, v[c]);
                    }
                    if (two && cb + TC_SUB * (u + 1) + c < p.nc) {
                        mn = fminf(mn, v2[c]);
                        mx = fmaxf(mx, v2[c]);
                    }
                }
            }
            float lo, hi;
            if (p.sym) {
                const float m = fmaxf(fabsf(mn), fabsf(mx));
                lo = -m;
                hi = m;
            } else {
                lo = fminf(mn, 0.f);
                hi = fmaxf(mx, 0.f);
            }
            float z;
            group_grid<BITS>(lo, hi, p.sym, st.s, z);
            st.inv_s = __frcp_rn(st.s);
            st.qlo = -z;
            st.qhi = (float)MAXQ - z;
            if (row_ok) {
                const long long gi = (p.c0 + cb) / p.g;
                p.scales[gi * p.d_out + row] = __float2half_rn(st.s);
                p.zeros_u8[gi * p.d_out + row] = (uint8_t)(int)z;
            }
        }
        // the 16 rounding steps; each error pushed into t's later columns and into t+1
        float e[TC_SUB], cnext[TC_SUB];
#pragma unroll
        for (int c = 0; c < TC_SUB; ++c) cnext[c] = 0.f;
        const float* uns = un + t * TC_SUB * TC_UNW;
#pragma unroll
        for (int c = 0; c < TC_SUB; ++c) {
            finite = finite && isfinite(w[c]);
            const float r = fminf(fmaxf(rintf(w[c] * st.inv_s), st.qlo), st.qhi);
            const float d = (cb + c < p.nc) ? fmaf(-r, st.s, w[c]) : 0.f;
            const unsigned code = (cb + c < p.nc) ? ((unsigned)(int)(r - st.qlo) & MAXQ) : 0u;
            bits_acc |= (unsigned long long)code << nbits;
            nbits += BITS;
            if (nbits >= 32) {
                if (row_ok && word < wend) p.qweight[word * p.d_out + row] = (int32_t)(uint32_t)bits_acc;
                bits_acc >>= 32;
                nbits -= 32;
                ++word;
            }
            const float4* ur = reinterpret_cast<const float4*>(uns + c * TC_UNW);
#pragma unroll
            for (int q = 0; q < TC_UNW / 4; ++q) {
                const float4 u4 = ur[q];
                const float uv[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int c2 = 4 * q + k;
                    if (c2 < TC_SUB) {
                        if (c2 > c) w[c2] = fmaf(-d, uv[k], w[c2]);
                    } else {
                        cnext[c2 - TC_SUB] = fmaf(-d, uv[k], cnext[c2 - TC_SUB]);
                    }
                }
            }
            e[c] = d * invd[cb + c];
        }
        // errors: per-row sum of squares, bf16 split to global, -e tf32 split as the A operand
        uint8_t* ah = sm + TCS_A + (t & 1) * 32768;
        uint8_t* al = ah + 16384;
#pragma unroll
        for (int c = 0; c < TC_SUB; ++c) {
            esum = fmaf(e[c], e[c], esum);
            float h, l;
            split_tf32(-e[c], h, l);
            *reinterpret_cast<float*>(ah + sw128_off(tid, c)) = h;
            *reinterpret_cast<float*>(al + sw128_off(tid, c)) = l;
        }
        if (row_ok) {   // 32-byte aligned: e_ld even, e_col0 and cb multiples of 16
            uint32_t hw[TC_SUB / 2], lw[TC_SUB / 2];
#pragma unroll
            for (int c = 0; c < TC_SUB; c += 2) {
                uint16_t h0, l0, h1, l1;
                split_bf16(e[c], h0, l0);
                split_bf16(e[c + 1], h1, l1);
                hw[c / 2] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                lw[c / 2] = (uint32_t)l0 | ((uint32_t)l1 << 16);
            }
            uint4* eh = reinterpret_cast<uint4*>(p.E_hi + row * p.e_ld + p.e_col0 + cb);
            uint4* el = reinterpret_cast<uint4*>(p.E_lo + row * p.e_ld + p.e_col0 + cb);
            eh[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            eh[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
            el[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            el[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
        }
        fence_proxy_async_smem();
        __syncthreads();
        const int n0 = TC_SUB * (t + 2);   // first column the product updates
        if (tid == 0 && t + 2 < TC_NSUB && n0 < p.nc) {
            tc_fence_after();
            const uint32_t a_hi = smem_u32(ah), a_lo = smem_u32(al);
            const uint32_t b_hi = smem_u32(sm + TCS_BH), b_lo = smem_u32(sm + TCS_BL);
            const uint32_t idesc = make_idesc(2u, TC_ROWS, CB - n0);
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                const uint32_t ao = (uint32_t)(ks * 32);
                const uint32_t bo = (uint32_t)((t >> 1) * 16384 + n0 * 128 + (t & 1) * 64 + ks * 32);
                const uint32_t acc0 = (t == 0 && ks == 0) ? 0u : 1u;
                umma_tf32(tmem + (uint32_t)n0, desc_sw128_kmajor(a_hi + ao), desc_sw128_kmajor(b_hi + bo), idesc, acc0);
                umma_tf32(tmem + (uint32_t)(CB + n0), desc_sw128_kmajor(a_hi + ao), desc_sw128_kmajor(b_lo + bo), idesc,
                          acc0);
                umma_tf32(tmem + (uint32_t)(CB + n0), desc_sw128_kmajor(a_lo + ao), desc_sw128_kmajor(b_hi + bo), idesc,
                          1u);
            }
            umma_commit(&bar_mma[t & 1]);
        }
#pragma unroll
        for (int c = 0; c < TC_SUB; ++c) wcur[c] = wnext[c] + cnext[c];
    }
    (void)FULL;
    if (!finite && row_ok) record_status(GPTQ_ERR_NONFINITE, row);
    if (row_ok && p.err_sq) p.err_sq[row] = (p.first_block ? 0.f : p.err_sq[row]) + esum;
    if (row_ok && ok && nbits > 0 && word < wend) p.qweight[word * p.d_out + row] = (int32_t)(uint32_t)bits_acc;
    // the products still in flight (the main loop waited for those up to nsub - 3) finish
    // before the tensor memory is released; each commit is waited for at most once past this
    for (int t = nsub - 2; t < nsub; ++t)
        if (t >= 0) (void)wait_mma(t);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// Per layer, for every 128-column block b (c0 = 128 b): the normalised U rows of each
// sub-block s, un[b][s][c][c2] = U[c0+16s+c, c0+16s+c2] / U[c0+16s+c, c0+16s+c] for the
// sub-block's later columns (c2 < 16, c2 > c) and the next sub-block's (c2 >= 16), 0
// elsewhere; and inv_d[c] = 1 / U_cc.
__global__ void tc_un_prep_kernel(const float* __restrict__ U, long long d, float* __restrict__ un,
                                  float* __restrict__ inv_d) {
    const int b = blockIdx.x;
    const long long c0 = (long long)b * CB;
    const int nc = (int)min((long long)CB, d - c0);
    for (int e = threadIdx.x; e < TC_UN; e += blockDim.x) {
        const int s = e / (TC_SUB * TC_UNW), c = (e / TC_UNW) % TC_SUB, c2 = e % TC_UNW;
        const int i = TC_SUB * s + c, j = TC_SUB * s + c2;
        float v = 0.f;
        if (c2 > c && i < nc && j < nc && j < CB) v = __fdiv_rn(U[(c0 + i) * d + c0 + j], U[(c0 + i) * d + c0 + i]);
        un[(long long)b * TC_UN + e] = v;
    }
    for (int c = threadIdx.x; c < nc; c += blockDim.x) inv_d[c0 + c] = __frcp_rn(U[(c0 + c) * d + c0 + c]);
}

// Per layer: the U^T tile of every block, tf32 split: tile[b][n][k] = U[c0+k, c0+n] (0 past d;
// U is upper triangular, so 0 for n < k).  One CTA per (block, 32 K-columns of the tile).
__global__ void tc_ut_prep_kernel(const float* __restrict__ U, long long d, float* __restrict__ t_hi,
                                  float* __restrict__ t_lo) {
    __shared__ float tile[32][CB + 1];   // tile[k - k0][n] for 32 consecutive k
    const int b = blockIdx.y, k0 = 32 * blockIdx.x;
    const long long c0 = (long long)b * CB;
    const int nc = (int)min((long long)CB, d - c0);
    for (int e = threadIdx.x; e < 32 * CB; e += blockDim.x) {   // read rows k of U, coalesced along n
        const int kk = e / CB, n = e % CB, k = k0 + kk;
        tile[kk][n] = (k < nc && n < nc && n >= k) ? U[(c0 + k) * d + c0 + n] : 0.f;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * CB; e += blockDim.x) {   // write tile rows n, 32 k each
        const int n = e / 32, kk = e % 32;
        float h, l;
        split_tf32(tile[kk][n], h, l);
        const long long off = ((long long)b * CB + n) * CB + k0 + kk;
        t_hi[off] = h;
        t_lo[off] = l;
    }
}

}  // namespace gq
