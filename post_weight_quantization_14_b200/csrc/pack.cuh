// Bit packing of b-bit codes into int32 words and dequantization.
// Layout (chosen; the pages fix only the code range and the group semantics):
// each row's codes form a little-endian stream, code j at bits j*b .. j*b+b-1,
// cut into 32-bit words; a 3-bit code may straddle two words.
#pragma once
#include "common.cuh"

namespace gq {

// One thread per output word.  layout 0: out[r*nwords + k]; layout 1: out[k*rows + r].
__global__ void pack_int_kernel(const uint8_t* __restrict__ codes, long long rows, long long cols,
                                int bits, int layout, int32_t* __restrict__ out) {
    const long long nwords = (cols * bits + 31) / 32;
    const long long total = rows * nwords;
    const uint32_t mask = (1u << bits) - 1u;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        long long r, k;
        if (layout == 1) {   // consecutive threads -> consecutive rows of one word index
            k = idx / rows;
            r = idx % rows;
        } else {
            r = idx / nwords;
            k = idx % nwords;
        }
        const long long bit0 = k * 32;
        const long long j0 = bit0 / bits;
        const long long j1 = min(cols - 1, (bit0 + 31) / bits);
        unsigned long long acc = 0;
        for (long long j = j0; j <= j1; ++j) {
            const long long sh = j * bits - bit0 + 8;  // >= 6 since a code starts at most 2 bits early
            acc |= (unsigned long long)(codes[r * cols + j] & mask) << sh;
        }
        const int32_t word = (int32_t)(uint32_t)(acc >> 8);
        if (layout == 1)
            out[k * rows + r] = word;
        else
            out[r * nwords + k] = word;
    }
}

__device__ __forceinline__ uint32_t stream_code(const int32_t* words, long long word_stride, long long j,
                                                int bits) {
    // code j of a stream whose word k sits at words[k * word_stride]
    const long long bit = j * bits;
    const long long k = bit >> 5;
    const int sh = (int)(bit & 31);
    uint64_t v = (uint32_t)words[k * word_stride];
    if (sh + bits > 32) v |= (uint64_t)(uint32_t)words[(k + 1) * word_stride] << 32;
    return (uint32_t)(v >> sh) & ((1u << bits) - 1u);
}

// W_hat[o, c] = scale[g(c), o] * (q[o, c] - zero[g(c), o]); one thread per weight, row-major.
// g(c) = c / g, or g_idx[c] when a per-column group index is given (activation ordering);
// an index outside [0, n_groups) is recorded as GPTQ_ERR_INVALID_ARG and group 0 is used.
__global__ void dequant_kernel(const int32_t* __restrict__ qweight, const __half* __restrict__ scales,
                               const int32_t* __restrict__ qzeros, const int32_t* __restrict__ g_idx,
                               long long d_out, long long d_in, int bits, int g, int sym,
                               float* __restrict__ W_hat) {
    const long long total = d_out * d_in;
    const long long zwords = (d_out * bits + 31) / 32;
    const long long ng = (d_in + g - 1) / g;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long o = idx / d_in, c = idx % d_in;
        long long gi = c / g;
        if (g_idx) {
            gi = g_idx[c];
            if (gi < 0 || gi >= ng) {
                record_status(GPTQ_ERR_INVALID_ARG, c);
                gi = 0;
            }
        }
        const uint32_t q = stream_code(qweight + o, d_out, c, bits);
        const float s = __half2float(scales[gi * d_out + o]);
        float z;
        if (sym)
            z = (float)(1 << (bits - 1));
        else
            z = (float)stream_code(qzeros + gi * zwords, 1, o, bits);
        W_hat[idx] = s * ((float)q - z);
    }
}

}  // namespace gq
