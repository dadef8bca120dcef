// Host side of the column loop: workspace, the per-block launch sequence with the trailing
// updates (tutorial "阶段二": one trailing update per lazy block), and the activation-ordered
// variant.
#pragma once
#include "colloop.cuh"

namespace gqh {

struct QuantWs {
    float *Up, *inv_d, *row_scale, *row_zero;
    uint16_t *UT_hi, *UT_lo, *E_hi, *E_lo;   // bf16 splits (operands of the trailing updates)
    uint8_t* zeros_u8;
};

inline long long n_groups_of(long long d_in, int g) { return g < 0 ? 1 : (d_in + g - 1) / g; }

// Trailing updates are deferred within superblocks of SB_BLOCKS column blocks: after
// each block only the rest of its superblock is updated (K = 128); the columns past the
// superblock take one update with K = the superblock width when it ends.  The result is
// the per-block lazy update regrouped by associativity.
constexpr int SB_BLOCKS = 8;

inline long long superblock_cols(long long d_in) {
    return std::min<long long>((long long)SB_BLOCKS * gq::CB, ((d_in + gq::CB - 1) / gq::CB) * gq::CB);
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline size_t quant_ws_bytes(long long d_out, long long d_in, int g) {
    const long long nblk = (d_in + gq::CB - 1) / gq::CB;
    size_t b = 0;
    b += align256((size_t)nblk * gq::UP_BLOCK * 4);
    b += align256((size_t)d_in * 4);
    b += 2 * align256((size_t)d_in * d_in * 2);
    b += 2 * align256((size_t)d_out * superblock_cols(d_in) * 2);
    b += 2 * align256((size_t)d_out * 4);
    b += align256((size_t)n_groups_of(d_in, g) * d_out);
    return b;
}

inline QuantWs quant_ws_carve(void* ws, long long d_out, long long d_in, int g) {
    const long long nblk = (d_in + gq::CB - 1) / gq::CB;
    uint8_t* p = static_cast<uint8_t*>(ws);
    QuantWs w;
    auto take = [&](size_t bytes) {
        uint8_t* q = p;
        p += align256(bytes);
        return q;
    };
    w.Up = reinterpret_cast<float*>(take((size_t)nblk * gq::UP_BLOCK * 4));
    w.inv_d = reinterpret_cast<float*>(take((size_t)d_in * 4));
    w.UT_hi = reinterpret_cast<uint16_t*>(take((size_t)d_in * d_in * 2));
    w.UT_lo = reinterpret_cast<uint16_t*>(take((size_t)d_in * d_in * 2));
    w.E_hi = reinterpret_cast<uint16_t*>(take((size_t)d_out * superblock_cols(d_in) * 2));
    w.E_lo = reinterpret_cast<uint16_t*>(take((size_t)d_out * superblock_cols(d_in) * 2));
    w.row_scale = reinterpret_cast<float*>(take((size_t)d_out * 4));
    w.row_zero = reinterpret_cast<float*>(take((size_t)d_out * 4));
    w.zeros_u8 = take((size_t)n_groups_of(d_in, g) * d_out);
    return w;
}

template <int BITS>
cudaError_t quant_run_bits(float* W, const float* U, long long d_out, long long d_in, const gptq_config& cfg,
                           int32_t* qweight, __half* scales, int32_t* qzeros, float* err_sq, void* ws,
                           cudaStream_t st) {
    const int g = cfg.group_size;
    QuantWs w = quant_ws_carve(ws, d_out, d_in, g);
    const int nblk = (int)((d_in + gq::CB - 1) / gq::CB);
    {
        dim3 grid(gq::CB, nblk);
        {
            gqh::TimedScope ts__("up_prep", st);
            gq::up_prep_kernel<<<grid, 160, 0, st>>>(U, d_in, w.Up, w.inv_d);
        }
        GQ_TRY(cudaGetLastError());
        const unsigned nt = (unsigned)((d_in + gq::UTS - 1) / gq::UTS);
        {
            gqh::TimedScope ts__("ut_split", st);
            gq::ut_split_kernel<<<dim3(nt, nt), 256, 0, st>>>(U, d_in, w.UT_hi, w.UT_lo);
        }
        GQ_TRY(cudaGetLastError());
    }
    if (g < 0) {
        {
            gqh::TimedScope ts__("row_params", st);
            gq::row_params_kernel<BITS><<<(unsigned)((d_out + 7) / 8), 256, 0, st>>>(
                W, d_out, d_in, cfg.sym, w.row_scale, w.row_zero, scales, w.zeros_u8);
        }
        GQ_TRY(cudaGetLastError());
    }
    const int smem = (int)sizeof(gq::ColSmem);
    GQ_TRY(ensure_smem_attr(reinterpret_cast<const void*>(gq::colloop_kernel<BITS>), smem));
    const unsigned grid = (unsigned)((d_out + gq::CL_ROWS - 1) / gq::CL_ROWS);
    const long long sbw = superblock_cols(d_in);
    Mat eh{w.E_hi, (uint64_t)d_out, (uint64_t)sbw, (uint64_t)sbw};
    Mat el{w.E_lo, (uint64_t)d_out, (uint64_t)sbw, (uint64_t)sbw};
    Mat uh{w.UT_hi, (uint64_t)d_in, (uint64_t)d_in, (uint64_t)d_in};
    Mat ul{w.UT_lo, (uint64_t)d_in, (uint64_t)d_in, (uint64_t)d_in};
    // W[:, e:e+n] -= E[:, k0:k0+K] U[c0:c0+K, e:e+n]  (U^T split is the B operand)
    auto trailing = [&](long long e, long long ncols, int k0, long long c0, int K, const char* name) {
        gq::GemmArgs p = gemm_args((int)d_out, (int)ncols, K);
        p.a_col0 = k0;
        p.b_row0 = (int)e;
        p.b_col0 = (int)c0;
        p.alpha = -1.f;
        p.beta = 1.f;
        p.c_col0 = (int)e;
        p.write_c = 1;
        p.b_early = 1;   // U^T's split is made before the first column loop
        EpiMats o;
        o.c = Mat{W, (uint64_t)d_out, (uint64_t)d_in, (uint64_t)d_in};
        // few 128-wide tiles: 128x32 tiles spread the work over more SMs, within one wave.
        // bf16x3 products (16-bit operand splits) at the bf16 rate; segmented accumulation
        // (8 k-steps = 128 K per segment, cross products apart): the in-place fp32
        // accumulation of a K = 1024 update drifts by ~1e-5 relative, enough to move
        // near-tie rounding decisions of later columns.
        if (4 * ((d_out + gq::BM - 1) / gq::BM) * ((ncols + gq::CB - 1) / gq::CB) <= num_sms())
            return launch_gemm<gq::KIND_BF16X3, 4, 32, 8>(eh, el, uh, ul, o, p, 1, st, name);
        return launch_gemm<gq::KIND_BF16X3, 2, 128, 8>(eh, el, uh, ul, o, p, 1, st, name);
    };
    for (int b = 0; b < nblk; ++b) {
        const long long s0 = (long long)(b / SB_BLOCKS) * sbw;      // superblock columns
        const long long s1 = std::min<long long>(s0 + sbw, d_in);
        const int kin = (int)((long long)b * gq::CB - s0);                // block offset in it
        gq::ColArgs a{};
        a.W = W;
        a.d_out = d_out;
        a.d_in = d_in;
        a.c0 = b * gq::CB;
        a.nc = (int)std::min<long long>(gq::CB, d_in - a.c0);
        a.Up = w.Up + (long long)b * gq::UP_BLOCK;
        a.inv_d = w.inv_d;
        a.g = g;
        a.sym = cfg.sym;
        a.row_scale = w.row_scale;
        a.row_zero = w.row_zero;
        a.qweight = qweight;
        a.scales = scales;
        a.zeros_u8 = w.zeros_u8;
        a.E_hi = w.E_hi + kin;
        a.E_lo = w.E_lo + kin;
        a.e_ld = sbw;
        a.err_sq = err_sq;
        a.first_block = (b == 0);
        {
            gqh::TimedScope ts__("colloop", st);
            GQ_TRY(launch_pdl(gq::colloop_kernel<BITS>, dim3(grid), dim3(gq::CL_WARPS * 32), (size_t)smem, st,
                              (const gq::ColArgs)a));
        }
        const long long e = (long long)a.c0 + gq::CB;
        if (e < s1)   // the rest of this superblock
            GQ_TRY(trailing(e, s1 - e, kin, a.c0, gq::CB, "trailing_update"));
        if (e == s1 && s1 < d_in)   // superblock done: everything past it, K = its width
            GQ_TRY(trailing(s1, d_in - s1, 0, s0, (int)(s1 - s0), "trailing_update_sb"));
    }
    if (!cfg.sym && qzeros) {
        const long long ng = n_groups_of(d_in, g);
        const long long words = ng * ((d_out * BITS + 31) / 32);
        {
            gqh::TimedScope ts__("pack_zeros", st);
            gq::pack_int_kernel<<<(unsigned)std::min<long long>((words + 255) / 256, 4096), 256, 0, st>>>(
                w.zeros_u8, ng, d_out, BITS, 0, qzeros);
        }
        GQ_TRY(cudaGetLastError());
    }
    return cudaSuccess;
}

// Activation-ordered column loop: the workspace of the plain loop, then the gathered
// weights Wp, the permuted codes and the inverse permutation.
inline size_t act_quant_ws_bytes(long long d_out, long long d_in, int g, int bits) {
    const long long words = (d_in * bits + 31) / 32;
    return quant_ws_bytes(d_out, d_in, g) + align256((size_t)d_out * d_in * 4) +
           align256((size_t)words * d_out * 4) + align256((size_t)d_in * 4);
}

// Validate perm (rank = its inverse), gather W's columns into quantization order, run
// the unchanged column loop on them (scales, zeros and err_sq go straight to the
// caller's buffers: groups are in quantization order), then repack the codes in the
// original column order and write g_idx.
template <int BITS>
cudaError_t act_quant_run_bits(const float* W, const float* U, const int* perm, long long d_out, long long d_in,
                               const gptq_config& cfg, int32_t* qweight, __half* scales, int32_t* qzeros,
                               int32_t* g_idx, float* err_sq, void* ws, cudaStream_t st) {
    const long long words = (d_in * BITS + 31) / 32;
    uint8_t* p = static_cast<uint8_t*>(ws) + quant_ws_bytes(d_out, d_in, cfg.group_size);
    float* Wp = reinterpret_cast<float*>(p);
    p += align256((size_t)d_out * d_in * 4);
    int32_t* qw_perm = reinterpret_cast<int32_t*>(p);
    p += align256((size_t)words * d_out * 4);
    int* rank = reinterpret_cast<int*>(p);
    GQ_TRY(cudaMemsetAsync(rank, 0xFF, (size_t)d_in * sizeof(int), st));
    {
        gqh::TimedScope ts__("perm_invert", st);
        gq::perm_invert_kernel<<<(unsigned)((d_in + 255) / 256), 256, 0, st>>>(perm, d_in, rank);
    }
    GQ_TRY(cudaGetLastError());
    {
        gqh::TimedScope ts__("gather_cols", st);
        const size_t row_bytes = (size_t)d_in * sizeof(float);
        constexpr int kMaxRowBytes = 96 * 1024;   // two or more CTAs per SM
        if (row_bytes <= (size_t)kMaxRowBytes) {   // the attribute is a fixed upper bound for every width
            GQ_TRY(ensure_smem_attr(reinterpret_cast<const void*>(gq::gather_cols_smem_kernel), kMaxRowBytes));
            const long long per_sm = std::min<long long>(8, (200 * 1024) / row_bytes);
            gq::gather_cols_smem_kernel<<<(unsigned)std::min<long long>(d_out, per_sm * num_sms()), 256, row_bytes,
                                          st>>>(W, perm, d_out, d_in, Wp);
        } else {
            gq::gather_cols_kernel<<<(unsigned)std::min<long long>(d_out, 8192), 256, 0, st>>>(W, perm, d_out, d_in,
                                                                                          Wp);
        }
    }
    GQ_TRY(cudaGetLastError());
    GQ_TRY(quant_run_bits<BITS>(Wp, U, d_out, d_in, cfg, qw_perm, scales, qzeros, err_sq, ws, st));
    const long long items = std::max(words * d_out, d_in);
    {
        gqh::TimedScope ts__("unpermute_codes", st);
        gq::unpermute_codes_kernel<<<(unsigned)std::min<long long>((items + 255) / 256, 8192), 256, 0, st>>>(
            qw_perm, rank, d_out, d_in, BITS, cfg.group_size < 0 ? (int)d_in : cfg.group_size, qweight, g_idx);
    }
    return cudaGetLastError();
}

}  // namespace gqh
