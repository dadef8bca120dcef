// GPTQ column loop for one 128-column lazy block (tutorial "阶段二" greedy order and
// lazy batch updates, "阶段三" group-wise scale; group-size article for scale/zero).
//
// Rows are independent.  Eight lanes share one row; lane k of the row holds the
// block's columns k, k+8, ..., k+120 in registers (cyclic mapping keeps the per-step
// update work balanced across the lanes).  The block is walked in 16 "octs" of eight
// columns by a rolled loop: register slot 0 always holds the lane's column of the
// current oct and the slots shift down by one after each oct, so the loop body stays
// small (a fully unrolled 128-step loop thrashed the instruction cache).  Four phases
// of four octs carry 16, 12, 8 and 4 live slots.  Per oct, the row's 8 lanes gather the
// oct's 8 current values, and every lane then runs the oct's 8 rounding steps itself (the
// same operations in the same order, so all lanes agree exactly): for column c,
//   r = clamp(rint(w_c / s), -z, maxq - z);  d_c = w_c - s * r;
//   w_j -= d_c * U[c, j] / U[c, c]   for the later columns j of the oct;
// after the oct each lane applies the 8 errors d_c to its later slots in column order,
// which is e_c = d_c / U_cc pushed forward with row c of U.  The normalised rows of
// the block's 128x128 diagonal part of U are prepared once per layer and staged into
// shared memory by four bulk (TMA) copies per CTA, one per phase, each waited for just
// before its phase.
// At a group's first column the scale and zero come from the current values of the
// group's columns (min/max by an 8-lane shuffle reduction).
// At the end of the block the kernel writes the packed codes (qweight layout), the
// errors e = d / U_cc as a bf16 split (operand of the bf16x3 trailing tensor-core update)
// and the per-row sum of e^2.
#pragma once
#include "gemm_tc.cuh"
#include "pack.cuh"
#include "actorder.cuh"

namespace gq {

constexpr int CB = 128;                  // lazy block width
constexpr int LPR = 8;                   // lanes per row
constexpr int SLOTS = CB / LPR;          // register slots per lane
constexpr int RPW = 32 / LPR;            // rows per warp
constexpr int CL_WARPS = 4;
constexpr int CL_ROWS = CL_WARPS * RPW;  // rows per CTA
constexpr int UP_LD = 20;                // padded slot stride of one lane's row segment (16 used)
constexpr int UP_OCT = LPR * UP_LD;      // offset of a row's eight in-oct entries
constexpr int UP_ROW = UP_OCT + 8;       // floats per normalised U row
constexpr int UP_BLOCK = CB * UP_ROW;    // floats per block (86016 bytes)
constexpr int CODE_LD = 132;
constexpr int DV_LD = 129;
constexpr float kF16MinPos = 5.9604644775390625e-08f;  // 2^-24, smallest positive fp16

struct ColArgs {
    float* W;
    long long d_out, d_in;
    int c0, nc;
    const float* Up;      // normalised, quad-shifted U rows of this block, [128][UP_ROW]
    const float* inv_d;   // [d_in] 1 / U_cc
    int g, sym;
    const float* row_scale;
    const float* row_zero;
    int32_t* qweight;
    __half* scales;
    uint8_t* zeros_u8;
    uint16_t* E_hi;       // errors of this block: E[row * e_ld + col], bf16 split (bit patterns)
    uint16_t* E_lo;
    long long e_ld;
    float* err_sq;
    int first_block;
};

struct ColSmem {
    float up[UP_BLOCK];
    float dv[CL_ROWS][DV_LD];
    float invd[CB];
    uint8_t codes[CL_ROWS][CODE_LD];
    uint64_t bar[4];   // one per quarter of the staged rows (the 32 columns of one phase)
};

// Scale and zero of a group with grid range [lo, hi] (lo <= 0 <= hi, or -m..m).
template <int BITS>
__device__ __forceinline__ void group_grid(float lo, float hi, int sym, float& s, float& z) {
    constexpr int MAXQ = (1 << BITS) - 1;
    if (hi == lo) {
        s = 1.f;
    } else {
        s = __half2float(__float2half_rn(__fdiv_rn(hi - lo, (float)MAXQ)));
        if (s == 0.f) s = kF16MinPos;
    }
    if (sym)
        z = (float)(1 << (BITS - 1));
    else
        z = fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.f), (float)MAXQ);
}

struct QuadState {
    float s, inv_s, qlo, qhi;  // current group: scale, 1/scale, -zero, maxq - zero
};

// Octs [t0, t1) of the block with LIVE register slots in use.  Slot i of lane k holds
// column 8*(t + i) + k at oct t; the normalised U row of column c is stored shifted so
// that its entry for slot i is at offset i (zeros for columns at or before c).
// Per oct, the 8 lanes of a row first gather the oct's 8 current column values (one
// shuffle each, all independent), then every lane runs the oct's 8 rounding steps itself
// in registers (the same operations in the same order in all 8 lanes, so the results
// agree exactly), and finally applies the 8 errors to its remaining slots in column
// order.  The dependent chain of one rounding step has no shuffle in it.
template <int BITS, int LIVE>
__device__ __forceinline__ void run_octs(float (&wv)[SLOTS], int t0, int t1, QuadState& st, const ColArgs& p,
                                         ColSmem& S, int lane, int k, int rloc, long long row, bool row_ok) {
    constexpr unsigned FULL = 0xffffffffu;
    constexpr int MAXQ = (1 << BITS) - 1;
    const int g = p.g;
    const int base = lane & ~(LPR - 1);
#pragma unroll 1
    for (int t = t0; t < t1; ++t) {
        const int c8 = LPR * t;
        if (g > 0 && (c8 & (g - 1)) == 0) {
            const int gslots = g / LPR;
            float mn = INFINITY, mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < LIVE; ++i) {
                if (i < gslots) {
                    mn = fminf(mn, wv[i]);
                    mx = fmaxf(mx, wv[i]);
                }
            }
#pragma unroll
            for (int o = 1; o < LPR; o <<= 1) {
                mn = fminf(mn, __shfl_xor_sync(FULL, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
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
            if (k == 0 && row_ok) {
                const long long gi = (p.c0 + c8) / g;
                p.scales[gi * p.d_out + row] = __float2half_rn(st.s);
                p.zeros_u8[gi * p.d_out + row] = (uint8_t)(int)z;
            }
        }
        // the oct's columns c8 .. c8+7 as they stand (slot 0 of the row's 8 lanes)
        float v[LPR];
#pragma unroll
        for (int j = 0; j < LPR; ++j) v[j] = __shfl_sync(FULL, wv[0], base | j);
        // its 8 rounding steps, with the in-oct propagation v[m] -= d_j U[c8+j][c8+m]
        float dd[LPR];
        float my_r = 0.f, my_d = 0.f;
#pragma unroll
        for (int j = 0; j < LPR; ++j) {
            const float r = fminf(fmaxf(rintf(v[j] * st.inv_s), st.qlo), st.qhi);
            const float d = fmaf(-r, st.s, v[j]);
            dd[j] = d;
            my_r = (k == j) ? r : my_r;
            my_d = (k == j) ? d : my_d;
            const float* urow = S.up + (c8 + j) * UP_ROW + UP_OCT;   // U[c8+j][c8+m] / U[c8+j][c8+j]
            const float4 ua = *reinterpret_cast<const float4*>(urow);
            const float4 ub = *reinterpret_cast<const float4*>(urow + 4);
            const float uo[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
#pragma unroll
            for (int m = j + 1; m < LPR; ++m) v[m] = fmaf(-d, uo[m], v[m]);
        }
        // the errors applied to this lane's later slots, in column order
#pragma unroll
        for (int j = 0; j < LPR; ++j) {
            const float4* u = reinterpret_cast<const float4*>(S.up + (c8 + j) * UP_ROW + k * UP_LD);
#pragma unroll
            for (int q = 0; q < LIVE / 4; ++q) {
                const float4 uu = u[q];
                if (4 * q + 0 > 0) wv[4 * q + 0] = fmaf(-dd[j], uu.x, wv[4 * q + 0]);
                wv[4 * q + 1] = fmaf(-dd[j], uu.y, wv[4 * q + 1]);
                wv[4 * q + 2] = fmaf(-dd[j], uu.z, wv[4 * q + 2]);
                wv[4 * q + 3] = fmaf(-dd[j], uu.w, wv[4 * q + 3]);
            }
        }
        S.codes[rloc][c8 + k] = (uint8_t)(int)(my_r - st.qlo);
        S.dv[rloc][c8 + k] = my_d;
#pragma unroll
        for (int i = 0; i < LIVE - 1; ++i) wv[i] = wv[i + 1];
        wv[LIVE - 1] = 0.f;
    }
}

template <int BITS>
__global__ void __launch_bounds__(CL_WARPS * 32) colloop_kernel(const ColArgs p) {
    extern __shared__ __align__(128) uint8_t cl_raw[];
    ColSmem& S = *reinterpret_cast<ColSmem*>(cl_raw);
    constexpr unsigned FULL = 0xffffffffu;
    constexpr int MAXQ = (1 << BITS) - 1;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = lane & (LPR - 1);
    const int rloc = warp * RPW + lane / LPR;
    const long long row = (long long)blockIdx.x * CL_ROWS + rloc;
    const bool row_ok = row < p.d_out;

    if (tid == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) mbar_init(&S.bar[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    // The staged U rows and 1/U_cc come from the layer's preparation kernels, which finished
    // before the grid this one waits for began (every grid of the sequence lets its dependent
    // start only after its own wait), so they are read before the wait: the copies overlap
    // the tail of the preceding trailing update.  W, which that update writes, is read after.
    if (tid == 0) {   // rows 32i .. 32i+31 (phase i's octs) complete barrier i
        constexpr uint32_t chunk = UP_BLOCK * 4 / 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            mbar_arrive_expect_tx(&S.bar[i], chunk);
            bulk_g2s(reinterpret_cast<uint8_t*>(S.up) + i * chunk,
                     reinterpret_cast<const uint8_t*>(p.Up) + i * chunk, chunk, &S.bar[i]);
        }
    }
    for (int c = tid; c < CB; c += blockDim.x) S.invd[c] = (c < p.nc) ? p.inv_d[p.c0 + c] : 0.f;
    pdl_wait();
    pdl_trigger();

    float wv[SLOTS];
    {
        const float* wrow = p.W + row * p.d_in + p.c0;
        bool finite = true;
#pragma unroll
        for (int t = 0; t < SLOTS; ++t) {
            const int col = k + LPR * t;
            float v = 0.f;
            if (row_ok && col < p.nc) v = wrow[col];
            finite = finite && isfinite(v);
            wv[t] = v;
        }
        if (!finite) record_status(GPTQ_ERR_NONFINITE, row);
    }

    float s = 1.f, inv_s = 1.f, qlo = 0.f, qhi = (float)MAXQ;
    if (p.g < 0 && row_ok) {
        const float z = p.row_zero[row];
        s = p.row_scale[row];
        inv_s = __frcp_rn(s);
        qlo = -z;
        qhi = (float)MAXQ - z;
    }
    const bool ok = mbar_wait(&S.bar[0], 0, -1 - (long long)blockIdx.x);
    __syncthreads();
    if (!ok) return;
    // the later quarters are waited for just before their phase (each warp decides as one,
    // so a warp never splits across a shuffle)
    auto staged = [&](int i) { return __all_sync(FULL, mbar_wait(&S.bar[i], 0, -1 - (long long)blockIdx.x)); };

    QuadState st{s, inv_s, qlo, qhi};
    run_octs<BITS, 16>(wv, 0, 4, st, p, S, lane, k, rloc, row, row_ok);
    if (!staged(1)) return;
    run_octs<BITS, 12>(wv, 4, 8, st, p, S, lane, k, rloc, row, row_ok);
    if (!staged(2)) return;
    run_octs<BITS, 8>(wv, 8, 12, st, p, S, lane, k, rloc, row, row_ok);
    if (!staged(3)) return;
    run_octs<BITS, 4>(wv, 12, 16, st, p, S, lane, k, rloc, row, row_ok);
    __syncwarp();

    // errors of the block (operand of the trailing update) and per-row sum of e^2; the
    // warp's rows are independent, so their loads, stores and reductions interleave
    const long long wrow0 = (long long)blockIdx.x * CL_ROWS + warp * RPW;
    float acc[RPW];
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
        const long long rw = wrow0 + rr;
        const int rl = warp * RPW + rr;
        acc[rr] = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int col = lane + 32 * q;
            const float e = S.dv[rl][col] * S.invd[col];
            acc[rr] = fmaf(e, e, acc[rr]);
            if (rw < p.d_out) {
                uint16_t h, l;
                split_bf16(e, h, l);
                p.E_hi[rw * p.e_ld + col] = h;
                p.E_lo[rw * p.e_ld + col] = l;
            }
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
#pragma unroll
        for (int rr = 0; rr < RPW; ++rr) acc[rr] += __shfl_xor_sync(FULL, acc[rr], o);
    }
    if (lane < RPW && p.err_sq) {
        float mine = acc[0];
#pragma unroll
        for (int rr = 1; rr < RPW; ++rr) mine = (lane == rr) ? acc[rr] : mine;
        const long long rw = wrow0 + lane;
        if (rw < p.d_out) p.err_sq[rw] = (p.first_block ? 0.f : p.err_sq[rw]) + mine;
    }

    // packed codes: word w of this block's stream for each of the warp's 8 rows
    const int nwb = (p.nc * BITS + 31) / 32;
    const long long wbase = (long long)p.c0 * BITS / 32;
    for (int idx = lane; idx < RPW * nwb; idx += 32) {
        const int rr = idx % RPW, w = idx / RPW;
        const long long rw = wrow0 + rr;
        if (rw >= p.d_out) continue;
        const int rl = warp * RPW + rr;
        const int bit0 = w * 32;
        const int j0 = bit0 / BITS, j1 = min(p.nc - 1, (bit0 + 31) / BITS);
        unsigned long long acc = 0;
        for (int j = j0; j <= j1; ++j)
            acc |= (unsigned long long)(S.codes[rl][j] & MAXQ) << (j * BITS - bit0 + 8);
        p.qweight[(wbase + w) * p.d_out + rw] = (int32_t)(uint32_t)(acc >> 8);
    }
}

// Normalised, lane-permuted, oct-shifted rows of each 128x128 diagonal block of U:
// Up[b][c][k*UP_LD + i] = U[c0+c, c0+j] / U[c0+c, c0+c] with j = k + 8*(c/8 + i) for j > c
// (0 otherwise), followed by the row's in-oct entries Up[b][c][UP_OCT + m] (the same value
// for j = 8*(c/8) + m), and inv_d[c] = 1 / U[c, c].
__global__ void up_prep_kernel(const float* __restrict__ U, long long d, float* __restrict__ Up,
                               float* __restrict__ inv_d) {
    const int b = blockIdx.y, c = blockIdx.x;
    const long long c0 = (long long)b * CB;
    const int nc = (int)min((long long)CB, d - c0);
    const float ucc = (c < nc) ? U[(c0 + c) * d + c0 + c] : 1.f;
    float* dst = Up + ((long long)b * CB + c) * UP_ROW;
    for (int e = threadIdx.x; e < UP_ROW; e += blockDim.x) {
        const int kk = e / UP_LD, i = e % UP_LD;
        const bool oct = e >= UP_OCT;
        const int j = oct ? LPR * (c / LPR) + (e - UP_OCT) : kk + LPR * ((c / LPR) + i);
        float v = 0.f;
        if ((oct || i < SLOTS) && c < nc && j < nc && j > c) v = __fdiv_rn(U[(c0 + c) * d + c0 + j], ucc);
        dst[e] = v;
    }
    if (threadIdx.x == 0 && c < nc) inv_d[c0 + c] = __frcp_rn(ucc);
}

// UT[j, i] = bf16 split of U[i, j] for the 64x64 tiles on or above the diagonal of U.
// 256 threads per tile: four float4 loads each (all issued first) into a padded tile, then
// 16-byte stores of eight consecutive bf16 values of a UT row per array.  d % 8 == 0.
constexpr int UTS = 64;
__global__ void __launch_bounds__(256) ut_split_kernel(const float* __restrict__ U, long long d,
                                                       uint16_t* __restrict__ UT_hi, uint16_t* __restrict__ UT_lo) {
    __shared__ float tile[UTS][UTS + 1];
    const long long bi = blockIdx.y, bj = blockIdx.x;  // tile of U
    if (bi > bj) return;
    float4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = threadIdx.x + 256 * q, r = e >> 4, c = (e & 15) * 4;
        const long long i = bi * UTS + r, j = bj * UTS + c;
        v[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < d && j < d) v[q] = *reinterpret_cast<const float4*>(U + i * d + j);   // d % 4 == 0
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = threadIdx.x + 256 * q, r = e >> 4, c = (e & 15) * 4;
        tile[r][c] = v[q].x;
        tile[r][c + 1] = v[q].y;
        tile[r][c + 2] = v[q].z;
        tile[r][c + 3] = v[q].w;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 2; ++q) {   // UT row jr of the tile, UT columns ir0 .. ir0 + 7
        const int e = threadIdx.x + 256 * q, jr = e >> 3, ir0 = (e & 7) * 8;
        const long long j = bj * UTS + jr, i0 = bi * UTS + ir0;
        if (j < d && i0 < d) {   // d % 8 == 0: the eight columns are wholly inside
            uint32_t h[4], l[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                uint16_t h0, l0, h1, l1;
                split_bf16(tile[ir0 + 2 * p][jr], h0, l0);
                split_bf16(tile[ir0 + 2 * p + 1][jr], h1, l1);
                h[p] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                l[p] = (uint32_t)l0 | ((uint32_t)l1 << 16);
            }
            *reinterpret_cast<uint4*>(UT_hi + j * d + i0) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4*>(UT_lo + j * d + i0) = make_uint4(l[0], l[1], l[2], l[3]);
        }
    }
}

// group_size = -1: one scale/zero per row from the whole original row.
template <int BITS>
__global__ void row_params_kernel(const float* __restrict__ W, long long d_out, long long d_in, int sym,
                                  float* __restrict__ row_scale, float* __restrict__ row_zero,
                                  __half* __restrict__ scales, uint8_t* __restrict__ zeros_u8) {
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= d_out) return;
    float mn = INFINITY, mx = -INFINITY;
    bool finite = true;
    for (long long c = lane; c < d_in; c += 32) {
        const float v = W[row * d_in + c];
        finite = finite && isfinite(v);
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
    }
    for (int o = 16; o; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (!finite) record_status(GPTQ_ERR_NONFINITE, row);
    if (lane == 0) {
        float lo, hi;
        if (sym) {
            const float m = fmaxf(fabsf(mn), fabsf(mx));
            lo = -m;
            hi = m;
        } else {
            lo = fminf(mn, 0.f);
            hi = fmaxf(mx, 0.f);
        }
        float s, z;
        group_grid<BITS>(lo, hi, sym, s, z);
        row_scale[row] = s;
        row_zero[row] = z;
        scales[row] = __float2half_rn(s);
        zeros_u8[row] = (uint8_t)(int)z;
    }
}

}  // namespace gq
