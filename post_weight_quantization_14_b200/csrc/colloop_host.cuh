// Host side of the column loop: workspace, the per-block launch sequence with the trailing
// updates (tutorial "阶段二": one trailing update per lazy block), and the activation-ordered
// variant.
#pragma once
#include "colloop_tc.cuh"

namespace gqh {

struct QuantWs {
    float *Up, *inv_d, *row_scale, *row_zero;
    float *un, *tb_hi, *tb_lo;                // tensor-core column loop: diagonal 16x16 blocks, U^T tiles
    uint16_t *UT_hi, *UT_lo, *E_hi, *E_lo;   // bf16 splits (operands of the trailing updates)
    uint8_t* zeros_u8;
};

inline long long n_groups_of(long long d_in, int g) { return g < 0 ? 1 : (d_in + g - 1) / g; }

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline size_t quant_ws_bytes(long long d_out, long long d_in, int g) {
    const long long nblk = (d_in + gq::CB - 1) / gq::CB;
    size_t b = 0;
    b += align256((size_t)nblk * gq::UP_BLOCK * 4);
    b += align256((size_t)d_in * 4);
    b += align256((size_t)nblk * gq::TC_UN * 4);
    b += 2 * align256((size_t)nblk * gq::CB * gq::CB * 4);
    b += 2 * align256((size_t)d_in * d_in * 2);
    b += 2 * align256((size_t)d_out * std::min<long long>(2 * gq::CB, nblk * gq::CB) * 2);
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
    w.un = reinterpret_cast<float*>(take((size_t)nblk * gq::TC_UN * 4));
    w.tb_hi = reinterpret_cast<float*>(take((size_t)nblk * gq::CB * gq::CB * 4));
    w.tb_lo = reinterpret_cast<float*>(take((size_t)nblk * gq::CB * gq::CB * 4));
    w.UT_hi = reinterpret_cast<uint16_t*>(take((size_t)d_in * d_in * 2));
    w.UT_lo = reinterpret_cast<uint16_t*>(take((size_t)d_in * d_in * 2));
    w.E_hi = reinterpret_cast<uint16_t*>(take((size_t)d_out * std::min<long long>(2 * gq::CB, nblk * gq::CB) * 2));
    w.E_lo = reinterpret_cast<uint16_t*>(take((size_t)d_out * std::min<long long>(2 * gq::CB, nblk * gq::CB) * 2));
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
        {
            gqh::TimedScope ts__("tc_un_prep", st);
            gq::tc_un_prep_kernel<<<(unsigned)nblk, 256, 0, st>>>(U, d_in, w.un, w.inv_d);
        }
        GQ_TRY(cudaGetLastError());
        {
            gqh::TimedScope ts__("tc_ut_prep", st);
            gq::tc_ut_prep_kernel<<<dim3(gq::CB / 32, (unsigned)nblk), 256, 0, st>>>(U, d_in, w.tb_hi, w.tb_lo);
        }
        GQ_TRY(cudaGetLastError());
        dim3 tb(32, 8), g2((unsigned)((d_in + 31) / 32), (unsigned)((d_in + 31) / 32));
        {
            gqh::TimedScope ts__("ut_split", st);
            gq::ut_split_kernel<<<g2, tb, 0, st>>>(U, d_in, w.UT_hi, w.UT_lo);
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
    GQ_TRY(ensure_smem_attr(reinterpret_cast<const void*>(gq::colloop_tc_kernel<BITS>), gq::TC_SMEM));
    const unsigned grid = (unsigned)((d_out + gq::TC_ROWS - 1) / gq::TC_ROWS);
    CUtensorMap m_tbh, m_tbl;
    if (!make_tmap_2d(&m_tbh, w.tb_hi, 4, (uint64_t)nblk * gq::CB, gq::CB, gq::CB, gq::TC_ROWS, 32) ||
        !make_tmap_2d(&m_tbl, w.tb_lo, 4, (uint64_t)nblk * gq::CB, gq::CB, gq::CB, gq::TC_ROWS, 32))
        return cudaErrorInvalidValue;
    // The block's errors go to one of two slots (block parity) of E, so the update of the
    // far columns by block b can still read them while block b+1 is quantized.
    const long long ecols = std::min<long long>(2 * gq::CB, (long long)nblk * gq::CB);
    Mat eh{w.E_hi, (uint64_t)d_out, (uint64_t)ecols, (uint64_t)ecols};
    Mat el{w.E_lo, (uint64_t)d_out, (uint64_t)ecols, (uint64_t)ecols};
    Mat uh{w.UT_hi, (uint64_t)d_in, (uint64_t)d_in, (uint64_t)d_in};
    Mat ul{w.UT_lo, (uint64_t)d_in, (uint64_t)d_in, (uint64_t)d_in};
    // W[:, e:e+n] -= E[:, k0:k0+128] U[c0:c0+128, e:e+n]  (U^T split is the B operand), bf16x3
    // products (16-bit operand splits) at the bf16 rate, accumulation segmented by 128 K with
    // the cross products apart
    auto trailing = [&](cudaStream_t s_, long long e, long long ncols, int k0, long long c0, const char* name,
                        int max_ctas, bool after) {
        gq::GemmArgs p = gemm_args((int)d_out, (int)ncols, gq::CB);
        p.a_col0 = k0;
        p.b_row0 = (int)e;
        p.b_col0 = (int)c0;
        p.alpha = -1.f;
        p.beta = 1.f;
        p.c_col0 = (int)e;
        p.write_c = 1;
        EpiMats o;
        o.c = Mat{W, (uint64_t)d_out, (uint64_t)d_in, (uint64_t)d_in};
        // few 128-wide tiles: 128x32 tiles spread the work over more SMs, within one wave
        if (4 * ((d_out + gq::BM - 1) / gq::BM) * ((ncols + gq::CB - 1) / gq::CB) <= num_sms())
            return launch_gemm<gq::KIND_BF16X3, 4, 32, 8>(eh, el, uh, ul, o, p, 1, s_, name, max_ctas, after);
        return launch_gemm<gq::KIND_BF16X3, 2, 128, 8>(eh, el, uh, ul, o, p, 1, s_, name, max_ctas, after);
    };
    // Streams: the chain (highest priority) runs, per block b, the column loop and then the
    // update of block b+1 by block b's errors; the far stream updates the columns past b+1.
    // Block b+1 also receives the far update of block b-1, which the chain waits for.
    FactStreams fs;
    if (!fact_streams(&fs)) return cudaErrorUnknown;
    cudaStream_t sc = fs.chain, sf = fs.far;
    cudaEvent_t ev_start = fs.ev[0], ev_col = fs.ev[1], ev_wide = fs.ev[2], ev_far = fs.ev[8], ev_chain = fs.ev[9];
    GQ_TRY(cudaEventRecord(ev_start, st));
    GQ_TRY(cudaStreamWaitEvent(sc, ev_start, 0));
    GQ_TRY(cudaStreamWaitEvent(sf, ev_start, 0));
    const int wide_ctas = std::max(1, num_sms() - (int)grid);   // leave the column loop its SMs
    bool wide_pending = false;
    for (int b = 0; b < nblk; ++b) {
        const int kin = ecols > gq::CB ? (b & 1) * gq::CB : 0;   // this block's slot in E
        gq::TcColArgs a{};
        a.W = W;
        a.d_out = d_out;
        a.d_in = d_in;
        a.c0 = b * gq::CB;
        a.nc = (int)std::min<long long>(gq::CB, d_in - a.c0);
        a.blk = b;
        a.un = w.un + (long long)b * gq::TC_UN;
        a.inv_d = w.inv_d;
        a.g = g;
        a.sym = cfg.sym;
        a.row_scale = w.row_scale;
        a.row_zero = w.row_zero;
        a.qweight = qweight;
        a.scales = scales;
        a.zeros_u8 = w.zeros_u8;
        a.E_hi = w.E_hi;
        a.E_lo = w.E_lo;
        a.e_ld = ecols;
        a.e_col0 = kin;
        a.err_sq = err_sq;
        a.first_block = (b == 0);
        {
            gqh::TimedScope ts__("colloop", sc);
            if (b == 0)   // follows the wait for the caller's stream
                GQ_TRY(launch_plain(gq::colloop_tc_kernel<BITS>, dim3(grid), dim3(gq::TC_ROWS), (size_t)gq::TC_SMEM,
                                    sc, m_tbh, m_tbl, (const gq::TcColArgs)a));
            else
                GQ_TRY(launch_pdl(gq::colloop_tc_kernel<BITS>, dim3(grid), dim3(gq::TC_ROWS), (size_t)gq::TC_SMEM,
                                  sc, m_tbh, m_tbl, (const gq::TcColArgs)a));
        }
        const long long e = (long long)a.c0 + gq::CB;
        if (e >= d_in) break;
        GQ_TRY(cudaEventRecord(ev_col, sc));
        const bool waited = wide_pending;
        if (wide_pending) GQ_TRY(cudaStreamWaitEvent(sc, ev_wide, 0));
        GQ_TRY(trailing(sc, e, std::min<long long>(gq::CB, d_in - e), kin, a.c0, "trailing_update", 0, waited));
        wide_pending = false;
        if (e + gq::CB < d_in) {
            GQ_TRY(cudaStreamWaitEvent(sf, ev_col, 0));
            GQ_TRY(trailing(sf, e + gq::CB, d_in - e - gq::CB, kin, a.c0, "trailing_update_wide", wide_ctas, true));
            GQ_TRY(cudaEventRecord(ev_wide, sf));
            wide_pending = true;
        }
    }
    GQ_TRY(cudaEventRecord(ev_far, sf));
    GQ_TRY(cudaEventRecord(ev_chain, sc));
    GQ_TRY(cudaStreamWaitEvent(st, ev_far, 0));
    GQ_TRY(cudaStreamWaitEvent(st, ev_chain, 0));
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
