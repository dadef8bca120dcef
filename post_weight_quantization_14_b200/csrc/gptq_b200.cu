// C ABI of the GPTQ layer-quantization library (declared in include/gptq_b200.h).
// Argument validation, workspace carving, status handling; all arithmetic runs in
// the kernels of the included headers.
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <set>
#include <string>
#include <tuple>
#include <vector>

#include "common.cuh"
#include "gemm_tc.cuh"
#include "hessian.cuh"
#include "chol_dag.cuh"
#include "pack.cuh"
#include "colloop_host.cuh"
#include "dqgemm.cuh"
#include "gptq2d.cuh"
#include "loss.cuh"

namespace gqh {

static thread_local char g_last_error[512] = "";

void set_last_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
}

// ---------------------------------------------------------------- per-launch timing
struct PendingLaunch {
    std::string name;
    cudaEvent_t a, b;
    cudaStream_t st;
};
struct TimelineEntry {
    std::string name;
    int stream;
    float t0, t1;   // ms from the first launch of the collected batch
};
static bool g_timing = false;
static std::vector<PendingLaunch> g_pending;
static std::vector<TimelineEntry> g_timeline;
static std::vector<cudaStream_t> g_timeline_streams;
static std::vector<cudaEvent_t> g_event_pool;
static std::map<std::string, std::pair<long long, double>> g_timing_acc;

static cudaEvent_t pooled_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

bool timing_on() { return g_timing; }

void timing_begin(const char* name, cudaStream_t st) {
    PendingLaunch p{name, pooled_event(), pooled_event(), st};
    cudaEventRecord(p.a, st);
    g_pending.push_back(p);
}

void timing_end(cudaStream_t st) {
    if (!g_pending.empty()) cudaEventRecord(g_pending.back().b, st);
}

static void timing_collect() {
    cudaDeviceSynchronize();
    const cudaEvent_t ref = g_pending.empty() ? nullptr : g_pending.front().a;
    for (auto& p : g_pending) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
            auto& acc = g_timing_acc[p.name];
            acc.first += 1;
            acc.second += ms;
        }
        float t0 = 0.f, t1 = 0.f;
        if (g_timeline.size() < 100000 && cudaEventElapsedTime(&t0, ref, p.a) == cudaSuccess &&
            cudaEventElapsedTime(&t1, ref, p.b) == cudaSuccess) {
            int si = -1;
            for (size_t k = 0; k < g_timeline_streams.size(); ++k)
                if (g_timeline_streams[k] == p.st) si = (int)k;
            if (si < 0) {
                si = (int)g_timeline_streams.size();
                g_timeline_streams.push_back(p.st);
            }
            g_timeline.push_back(TimelineEntry{p.name, si, t0, t1});
        }
        g_event_pool.push_back(p.a);
        g_event_pool.push_back(p.b);
    }
    g_pending.clear();
}

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Tensor maps depend only on (address, shape, box); the same buffers are reused by
// every block and every call, so encoded maps are cached (host memory only).
using TmapKey = std::tuple<uintptr_t, int, uint64_t, uint64_t, uint64_t, uint32_t, uint32_t>;
static std::map<TmapKey, CUtensorMap> g_tmap_cache;

static bool encode_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t rows, uint64_t cols,
                           uint64_t ld, uint32_t box_rows, uint32_t box_cols, bool swizzle = true);

bool make_tmap_2d_plain(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                        uint32_t box_rows, uint32_t box_cols) {
    return encode_tmap_2d(map, base, 4, rows, cols, ld, box_rows, box_cols, false);
}

bool make_tmap_2d_uncached(CUtensorMap* map, const void* base, int elem_bytes, uint64_t rows, uint64_t cols,
                           uint64_t ld, uint32_t box_rows, uint32_t box_cols) {
    return encode_tmap_2d(map, base, elem_bytes, rows, cols, ld, box_rows, box_cols);
}

bool make_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t rows, uint64_t cols,
                  uint64_t ld, uint32_t box_rows, uint32_t box_cols) {
    const TmapKey key{reinterpret_cast<uintptr_t>(base), elem_bytes, rows, cols, ld, box_rows, box_cols};
    auto it = g_tmap_cache.find(key);
    if (it != g_tmap_cache.end()) {
        *map = it->second;
        return true;
    }
    if (!encode_tmap_2d(map, base, elem_bytes, rows, cols, ld, box_rows, box_cols)) return false;
    if (g_tmap_cache.size() > 4096) g_tmap_cache.clear();
    g_tmap_cache.emplace(key, *map);
    return true;
}

int num_sms() {
    static int cache[128];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
    if (!cache[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        cache[dev] = v;
    }
    return cache[dev];
}

bool aux_stream(cudaStream_t* st, cudaEvent_t* ev0, cudaEvent_t* ev1) {
    static cudaStream_t streams[128];
    static cudaEvent_t events[128][2];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return false;
    if (!streams[dev]) {
        if (cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess) return false;
        if (cudaEventCreateWithFlags(&events[dev][0], cudaEventDisableTiming) != cudaSuccess) return false;
        if (cudaEventCreateWithFlags(&events[dev][1], cudaEventDisableTiming) != cudaSuccess) return false;
    }
    *st = streams[dev];
    *ev0 = events[dev][0];
    *ev1 = events[dev][1];
    return true;
}

bool fact_streams(FactStreams* fs) {
    static FactStreams cache[128];
    static bool made[128];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return false;
    if (!made[dev]) {
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return false;
        FactStreams f{};
        if (cudaStreamCreateWithPriority(&f.chain, cudaStreamNonBlocking, greatest) != cudaSuccess) return false;
        if (cudaStreamCreateWithPriority(&f.far, cudaStreamNonBlocking, least) != cudaSuccess) return false;
        if (cudaStreamCreateWithPriority(&f.inv, cudaStreamNonBlocking, least) != cudaSuccess) return false;
        for (auto& e : f.ev)
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
        cache[dev] = f;
        made[dev] = true;
    }
    *fs = cache[dev];
    return true;
}

cudaError_t ensure_smem_attr(const void* func, int bytes) {
    static std::set<std::tuple<const void*, int, int>> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const auto key = std::make_tuple(func, dev, bytes);
    if (done.count(key)) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.insert(key);
    return e;
}

static bool encode_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t rows, uint64_t cols,
                           uint64_t ld, uint32_t box_rows, uint32_t box_cols, bool swizzle) {
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return false;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (rows == 0 || cols == 0) return false;
    const CUtensorMapDataType dt =
        elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * (uint64_t)elem_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

static gptq_status fail(gptq_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return s;
}

static gptq_status cuda_fail(cudaError_t e, const char* where) {
    return fail(GPTQ_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static gptq_status check_config(const gptq_config* cfg) {
    if (!cfg) return fail(GPTQ_ERR_INVALID_ARG, "cfg is NULL");
    if (cfg->desc_act < 0 || cfg->desc_act > 2)
        return fail(GPTQ_ERR_INVALID_ARG, "desc_act must be 0, 1 (ascending) or 2 (descending) (got %d)", cfg->desc_act);
    if (!(cfg->bits == 2 || cfg->bits == 3 || cfg->bits == 4 || cfg->bits == 8))
        return fail(GPTQ_ERR_INVALID_ARG, "bits must be 2, 3, 4 or 8 (got %d)", cfg->bits);
    if (cfg->block_size != 128) return fail(GPTQ_ERR_INVALID_ARG, "block_size must be 128 (got %d)", cfg->block_size);
    const int g = cfg->group_size;
    if (!(g == -1 || (g >= 16 && g <= cfg->block_size && cfg->block_size % g == 0 && (g & (g - 1)) == 0)))
        return fail(GPTQ_ERR_INVALID_ARG, "group_size must be -1 or 16, 32, 64, 128 (got %d)", g);
    if (cfg->sym != 0 && cfg->sym != 1) return fail(GPTQ_ERR_INVALID_ARG, "sym must be 0 or 1");
    if (!(cfg->damp_rel >= 0.f) || cfg->damp_rel != cfg->damp_rel || cfg->damp_rel > 1e30f)
        return fail(GPTQ_ERR_INVALID_ARG, "damp_rel must be finite and >= 0");
    return GPTQ_OK;
}

static gptq_status read_status(cudaStream_t st, long long* index) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    unsigned long long v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, gq::g_status, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "read status");
    e = cudaMemcpyToSymbol(gq::g_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clear status");
    if (!v) return GPTQ_OK;
    const int code = (int)(v >> 48);
    long long idx = (long long)(v & 0xFFFFFFFFFFFFull);
    if (idx & 0x800000000000ll) idx |= ~0xFFFFFFFFFFFFll;  // sign-extend 48-bit index
    if (index) *index = idx;
    return fail((gptq_status)code, "device reported %s at index %lld", gptq_status_string((gptq_status)code), idx);
}

}  // namespace gqh

namespace gq {

// One thread waits on an mbarrier that nobody arrives at; the bounded wait records
// GPTQ_ERR_TIMEOUT and returns.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    mbar_init(&bar, 1);
    fence_mbar_init();
    (void)mbar_wait(&bar, 0, 0x7E57, limit_ns);
}

}  // namespace gq

using namespace gqh;

extern "C" {

void gptq_default_config(gptq_config* cfg) {
    if (!cfg) return;
    cfg->bits = 4;
    cfg->group_size = 128;
    cfg->sym = 0;
    cfg->block_size = 128;
    cfg->damp_rel = 0.01f;
    cfg->desc_act = 0;
}

const char* gptq_status_string(gptq_status s) {
    switch (s) {
        case GPTQ_OK: return "GPTQ_OK";
        case GPTQ_ERR_INVALID_ARG: return "GPTQ_ERR_INVALID_ARG";
        case GPTQ_ERR_UNSUPPORTED: return "GPTQ_ERR_UNSUPPORTED";
        case GPTQ_ERR_NOT_PD: return "GPTQ_ERR_NOT_PD";
        case GPTQ_ERR_NONFINITE: return "GPTQ_ERR_NONFINITE";
        case GPTQ_ERR_CUDA: return "GPTQ_ERR_CUDA";
        case GPTQ_ERR_TIMEOUT: return "GPTQ_ERR_TIMEOUT";
        case GPTQ_ERR_WORKSPACE: return "GPTQ_ERR_WORKSPACE";
    }
    return "GPTQ_ERR_UNKNOWN";
}

const char* gptq_last_error(void) { return g_last_error; }

int gptq_version(void) { return 100; }

size_t gptq_hessian_workspace_bytes(int64_t n, int64_t d_in, gptq_dtype xt) {
    if (n < 1 || d_in < 1) return 0;
    return hessian_ws_bytes(n, d_in, xt);
}

gptq_status gptq_hessian_accumulate(const void* X, gptq_dtype xt, int64_t n, int64_t d_in, float* H,
                                    int accumulate, void* ws, size_t ws_bytes, void* stream) {
    if (!X || !H) return fail(GPTQ_ERR_INVALID_ARG, "X and H must be non-NULL");
    if (xt != GPTQ_BF16 && xt != GPTQ_F32) return fail(GPTQ_ERR_INVALID_ARG, "unknown X dtype %d", (int)xt);
    if (n < 1 || n > (1ll << 30)) return fail(GPTQ_ERR_INVALID_ARG, "n out of range (%lld)", (long long)n);
    if (d_in < 8 || d_in > 65536 || d_in % 8) return fail(GPTQ_ERR_INVALID_ARG, "d_in must be a multiple of 8 in [8, 65536]");
    if (!aligned16(X) || !aligned16(H)) return fail(GPTQ_ERR_INVALID_ARG, "X and H must be 16-byte aligned");
    if (!ws || ws_bytes < hessian_ws_bytes(n, d_in, xt) || !aligned16(ws))
        return fail(GPTQ_ERR_WORKSPACE, "workspace needs %zu bytes", hessian_ws_bytes(n, d_in, xt));
    cudaError_t e = hessian_run(X, xt, n, d_in, H, accumulate ? 1 : 0, ws, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "hessian");
    return GPTQ_OK;
}

int64_t gptq_chol_schedule(int64_t T, int32_t* tasks, int64_t max_tasks) {
    if (T < 1 || T > 65536 / gq::NB + 1) return -1;
    const long long total = gq::dag_total_tasks((int)T);
    if (tasks) {
        gq::DagCursor cur{(int)T - 1, 0};
        for (long long t = 0; t < total && t < max_tasks; ++t) {
            const gq::DagTask k = gq::dag_decode((int)T, cur, t);
            tasks[4 * t + 0] = k.type;
            tasks[4 * t + 1] = k.a;
            tasks[4 * t + 2] = k.b;
            tasks[4 * t + 3] = k.c;
        }
    }
    return total;
}

size_t gptq_prepare_hinv_workspace_bytes(int64_t d_in) {
    if (d_in < 1) return 0;
    return hinv_ws_bytes(d_in);
}

static gptq_status prepare_hinv_common(const float* H, const int32_t* perm, int64_t d_in, float damp_rel, float* U,
                                       void* ws, size_t ws_bytes, int64_t* bad_col, float* lambda_out, void* stream) {
    if (!H || !U) return fail(GPTQ_ERR_INVALID_ARG, "H and U must be non-NULL");
    if (d_in < 8 || d_in > 65536 || d_in % 8) return fail(GPTQ_ERR_INVALID_ARG, "d_in must be a multiple of 8 in [8, 65536]");
    if (!(damp_rel >= 0.f) || damp_rel > 1e30f) return fail(GPTQ_ERR_INVALID_ARG, "damp_rel must be finite and >= 0");
    if (!aligned16(H) || !aligned16(U)) return fail(GPTQ_ERR_INVALID_ARG, "H and U must be 16-byte aligned");
    if (!ws || ws_bytes < hinv_ws_bytes(d_in) || !aligned16(ws))
        return fail(GPTQ_ERR_WORKSPACE, "workspace needs %zu bytes", hinv_ws_bytes(d_in));
    cudaStream_t st = (cudaStream_t)stream;
    long long idx = -1;
    gptq_status pre = read_status(st, &idx);  // clears any stale device status
    (void)pre;
    cudaError_t e = hinv_run(H, d_in, damp_rel, U, ws, st, perm);
    if (e != cudaSuccess) return cuda_fail(e, "prepare_hinv");
    idx = -1;
    gptq_status s = read_status(st, &idx);
    if (bad_col) *bad_col = (s == GPTQ_ERR_NOT_PD || s == GPTQ_ERR_NONFINITE) ? idx : -1;
    if (lambda_out) {
        HinvWs w = hinv_ws_carve(ws, d_in);
        float lam = 0.f;
        e = cudaMemcpy(&lam, w.scal, sizeof(float), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "read lambda");
        *lambda_out = lam;
    }
    return s;
}

}  // extern "C"

static gptq_status check_common(int64_t d_out, int64_t d_in, const float* W, const float* U) {
    if (d_out < 1 || d_out > (1ll << 30)) return fail(GPTQ_ERR_INVALID_ARG, "d_out out of range");
    if (d_in < 8 || d_in > 65536 || d_in % 8) return fail(GPTQ_ERR_INVALID_ARG, "d_in must be a multiple of 8 in [8, 65536]");
    if (!aligned16(W) || !aligned16(U)) return fail(GPTQ_ERR_INVALID_ARG, "W and U must be 16-byte aligned");
    return GPTQ_OK;
}

static gptq_status dequant_common(const int32_t* qweight, const uint16_t* scales, const int32_t* qzeros,
                                  const int32_t* g_idx, int64_t d_out, int64_t d_in, const gptq_config* cfg,
                                  float* W_hat, void* stream) {
    if (!cfg) return fail(GPTQ_ERR_INVALID_ARG, "cfg is NULL");
    if (!(cfg->bits == 2 || cfg->bits == 3 || cfg->bits == 4 || cfg->bits == 8))
        return fail(GPTQ_ERR_INVALID_ARG, "bits must be 2, 3, 4 or 8");
    if (!qweight || !scales || !W_hat) return fail(GPTQ_ERR_INVALID_ARG, "qweight, scales and W_hat must be non-NULL");
    if (cfg->sym ? (qzeros != nullptr) : (qzeros == nullptr))
        return fail(GPTQ_ERR_INVALID_ARG, "qzeros must be given iff asymmetric");
    if (d_out < 1 || d_in < 1) return fail(GPTQ_ERR_INVALID_ARG, "d_out and d_in must be >= 1");
    const int g = cfg->group_size < 0 ? (int)d_in : cfg->group_size;
    if (g < 1) return fail(GPTQ_ERR_INVALID_ARG, "group_size must be -1 or >= 1");
    const long long total = d_out * d_in;
    {
        gqh::TimedScope ts__("dequant", (cudaStream_t)stream);
        gq::dequant_kernel<<<(unsigned)std::min<long long>((total + 255) / 256, 16384), 256, 0, (cudaStream_t)stream>>>(
            qweight, reinterpret_cast<const __half*>(scales), qzeros, g_idx, d_out, d_in, cfg->bits, g, cfg->sym, W_hat);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "dequant");
    return GPTQ_OK;
}

static gptq_status prepare_hinv_async_common(const float* H, const int32_t* perm, int64_t d_in, float damp_rel,
                                             float* U, void* ws, size_t ws_bytes, float* lambda_dev, void* stream) {
    if (!H || !U) return fail(GPTQ_ERR_INVALID_ARG, "H and U must be non-NULL");
    if (d_in < 8 || d_in > 65536 || d_in % 8) return fail(GPTQ_ERR_INVALID_ARG, "d_in must be a multiple of 8 in [8, 65536]");
    if (!(damp_rel >= 0.f) || damp_rel > 1e30f) return fail(GPTQ_ERR_INVALID_ARG, "damp_rel must be finite and >= 0");
    if (!aligned16(H) || !aligned16(U)) return fail(GPTQ_ERR_INVALID_ARG, "H and U must be 16-byte aligned");
    if (lambda_dev && (reinterpret_cast<uintptr_t>(lambda_dev) & 3u))
        return fail(GPTQ_ERR_INVALID_ARG, "lambda_dev must be 4-byte aligned");
    if (!ws || ws_bytes < hinv_ws_bytes(d_in) || !aligned16(ws))
        return fail(GPTQ_ERR_WORKSPACE, "workspace needs %zu bytes", hinv_ws_bytes(d_in));
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = hinv_run(H, d_in, damp_rel, U, ws, st, perm);
    if (e != cudaSuccess) return cuda_fail(e, "prepare_hinv");
    if (lambda_dev) {
        HinvWs w = hinv_ws_carve(ws, d_in);
        e = cudaMemcpyAsync(lambda_dev, w.scal, sizeof(float), cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return cuda_fail(e, "lambda copy");
    }
    return GPTQ_OK;
}

extern "C" {

gptq_status gptq_prepare_hinv_async(const float* H, int64_t d_in, float damp_rel, float* U, void* ws,
                                    size_t ws_bytes, float* lambda_dev, void* stream) {
    return prepare_hinv_async_common(H, nullptr, d_in, damp_rel, U, ws, ws_bytes, lambda_dev, stream);
}

gptq_status gptq_prepare_hinv_permuted_async(const float* H, const int32_t* perm, int64_t d_in, float damp_rel,
                                             float* U, void* ws, size_t ws_bytes, float* lambda_dev, void* stream) {
    if (!perm) return fail(GPTQ_ERR_INVALID_ARG, "perm must be non-NULL");
    return prepare_hinv_async_common(H, perm, d_in, damp_rel, U, ws, ws_bytes, lambda_dev, stream);
}

gptq_status gptq_prepare_hinv(const float* H, int64_t d_in, float damp_rel, float* U, void* ws, size_t ws_bytes,
                              int64_t* bad_col, float* lambda_out, void* stream) {
    return prepare_hinv_common(H, nullptr, d_in, damp_rel, U, ws, ws_bytes, bad_col, lambda_out, stream);
}

gptq_status gptq_prepare_hinv_permuted(const float* H, const int32_t* perm, int64_t d_in, float damp_rel, float* U,
                                       void* ws, size_t ws_bytes, int64_t* bad_col, float* lambda_out, void* stream) {
    if (!perm) return fail(GPTQ_ERR_INVALID_ARG, "perm must be non-NULL");
    return prepare_hinv_common(H, perm, d_in, damp_rel, U, ws, ws_bytes, bad_col, lambda_out, stream);
}

gptq_status gptq_act_sum_accumulate(const void* X, gptq_dtype xt, int64_t n, int64_t d_in, double* act,
                                    int accumulate, void* stream) {
    if (!X || !act) return fail(GPTQ_ERR_INVALID_ARG, "X and act must be non-NULL");
    if (xt != GPTQ_BF16 && xt != GPTQ_F32) return fail(GPTQ_ERR_INVALID_ARG, "unknown X dtype %d", (int)xt);
    if (n < 1 || n > (1ll << 30)) return fail(GPTQ_ERR_INVALID_ARG, "n out of range (%lld)", (long long)n);
    if (d_in < 8 || d_in > 65536 || d_in % 8) return fail(GPTQ_ERR_INVALID_ARG, "d_in must be a multiple of 8 in [8, 65536]");
    if (!aligned16(X) || (reinterpret_cast<uintptr_t>(act) & 7u))
        return fail(GPTQ_ERR_INVALID_ARG, "X must be 16-byte and act 8-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    const unsigned grid = (unsigned)((d_in + gq::AS_COLS - 1) / gq::AS_COLS);
    {
        gqh::TimedScope ts__("act_sum", st);
        if (xt == GPTQ_BF16)
            gq::act_sum_kernel<true><<<grid, 256, 0, st>>>(X, n, d_in, accumulate ? 1 : 0, act);
        else
            gq::act_sum_kernel<false><<<grid, 256, 0, st>>>(X, n, d_in, accumulate ? 1 : 0, act);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "act_sum_accumulate");
    return GPTQ_OK;
}

gptq_status gptq_act_order(const double* act, int64_t d_in, int desc_act, int32_t* perm, int32_t* rank,
                           void* stream) {
    if (!act || !perm || !rank) return fail(GPTQ_ERR_INVALID_ARG, "act, perm and rank must be non-NULL");
    if (d_in < 1 || d_in > 65536) return fail(GPTQ_ERR_INVALID_ARG, "d_in must be in [1, 65536]");
    if (desc_act != 1 && desc_act != 2)
        return fail(GPTQ_ERR_INVALID_ARG, "desc_act must be 1 (ascending) or 2 (descending) (got %d)", desc_act);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(rank, 0, (size_t)d_in * sizeof(int32_t), st);
    if (e != cudaSuccess) return cuda_fail(e, "act_order");
    {
        gqh::TimedScope ts__("act_rank", st);
        const dim3 grid((unsigned)((d_in + gq::RK_THREADS - 1) / gq::RK_THREADS),
                        (unsigned)((d_in + gq::RK_CHUNK - 1) / gq::RK_CHUNK));
        gq::act_rank_kernel<<<grid, gq::RK_THREADS, 0, st>>>(act, d_in, desc_act == 2 ? 1 : 0, rank);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "act_order");
    {
        gqh::TimedScope ts__("act_perm", st);
        gq::act_perm_kernel<<<(unsigned)((d_in + 255) / 256), 256, 0, st>>>(rank, d_in, perm);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "act_order");
    return GPTQ_OK;
}

size_t gptq_quantize_workspace_bytes(int64_t d_out, int64_t d_in, const gptq_config* cfg) {
    if (d_out < 1 || d_in < 1 || !cfg) return 0;
    if (cfg->desc_act) return act_quant_ws_bytes(d_out, d_in, cfg->group_size, cfg->bits);
    return quant_ws_bytes(d_out, d_in, cfg->group_size);
}

gptq_status gptq_quantize_layer(float* W, const float* U, int64_t d_out, int64_t d_in, const gptq_config* cfg,
                                int32_t* qweight, uint16_t* scales, int32_t* qzeros, float* err_sq, void* ws,
                                size_t ws_bytes, void* stream) {
    gptq_status cs = check_config(cfg);
    if (cs != GPTQ_OK) return cs;
    if (cfg->desc_act)
        return fail(GPTQ_ERR_INVALID_ARG, "desc_act != 0: call gptq_quantize_layer_act_order with the permutation");
    if (!W || !U || !qweight || !scales) return fail(GPTQ_ERR_INVALID_ARG, "W, U, qweight and scales must be non-NULL");
    if (cfg->sym && qzeros) return fail(GPTQ_ERR_INVALID_ARG, "qzeros must be NULL for symmetric quantization");
    if (!cfg->sym && !qzeros) return fail(GPTQ_ERR_INVALID_ARG, "qzeros is required for asymmetric quantization");
    cs = check_common(d_out, d_in, W, U);
    if (cs != GPTQ_OK) return cs;
    const size_t need = quant_ws_bytes(d_out, d_in, cfg->group_size);
    if (!ws || ws_bytes < need || !aligned16(ws)) return fail(GPTQ_ERR_WORKSPACE, "workspace needs %zu bytes", need);
    cudaStream_t st = (cudaStream_t)stream;
    __half* sc = reinterpret_cast<__half*>(scales);
    cudaError_t e;
    switch (cfg->bits) {
        case 2: e = quant_run_bits<2>(W, U, d_out, d_in, *cfg, qweight, sc, qzeros, err_sq, ws, st); break;
        case 3: e = quant_run_bits<3>(W, U, d_out, d_in, *cfg, qweight, sc, qzeros, err_sq, ws, st); break;
        case 4: e = quant_run_bits<4>(W, U, d_out, d_in, *cfg, qweight, sc, qzeros, err_sq, ws, st); break;
        default: e = quant_run_bits<8>(W, U, d_out, d_in, *cfg, qweight, sc, qzeros, err_sq, ws, st); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "quantize_layer");
    return GPTQ_OK;
}

gptq_status gptq_quantize_layer_act_order(const float* W, const float* U, const int32_t* perm, int64_t d_out,
                                          int64_t d_in, const gptq_config* cfg, int32_t* qweight, uint16_t* scales,
                                          int32_t* qzeros, int32_t* g_idx, float* err_sq, void* ws, size_t ws_bytes,
                                          void* stream) {
    gptq_status cs = check_config(cfg);
    if (cs != GPTQ_OK) return cs;
    if (!cfg->desc_act) return fail(GPTQ_ERR_INVALID_ARG, "desc_act must be 1 or 2 for the activation-ordered loop");
    if (!W || !U || !perm || !qweight || !scales || !g_idx)
        return fail(GPTQ_ERR_INVALID_ARG, "W, U, perm, qweight, scales and g_idx must be non-NULL");
    if (cfg->sym && qzeros) return fail(GPTQ_ERR_INVALID_ARG, "qzeros must be NULL for symmetric quantization");
    if (!cfg->sym && !qzeros) return fail(GPTQ_ERR_INVALID_ARG, "qzeros is required for asymmetric quantization");
    cs = check_common(d_out, d_in, W, U);
    if (cs != GPTQ_OK) return cs;
    const size_t need = act_quant_ws_bytes(d_out, d_in, cfg->group_size, cfg->bits);
    if (!ws || ws_bytes < need || !aligned16(ws)) return fail(GPTQ_ERR_WORKSPACE, "workspace needs %zu bytes", need);
    cudaStream_t st = (cudaStream_t)stream;
    __half* sc = reinterpret_cast<__half*>(scales);
    cudaError_t e;
    switch (cfg->bits) {
        case 2: e = act_quant_run_bits<2>(W, U, perm, d_out, d_in, *cfg, qweight, sc, qzeros, g_idx, err_sq, ws, st); break;
        case 3: e = act_quant_run_bits<3>(W, U, perm, d_out, d_in, *cfg, qweight, sc, qzeros, g_idx, err_sq, ws, st); break;
        case 4: e = act_quant_run_bits<4>(W, U, perm, d_out, d_in, *cfg, qweight, sc, qzeros, g_idx, err_sq, ws, st); break;
        default: e = act_quant_run_bits<8>(W, U, perm, d_out, d_in, *cfg, qweight, sc, qzeros, g_idx, err_sq, ws, st); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "quantize_layer_act_order");
    return GPTQ_OK;
}

gptq_status gptq_pack_int(const uint8_t* codes, int64_t rows, int64_t cols, int bits, int layout, int32_t* packed,
                          void* stream) {
    if (!codes || !packed) return fail(GPTQ_ERR_INVALID_ARG, "codes and packed must be non-NULL");
    if (rows < 1 || cols < 1) return fail(GPTQ_ERR_INVALID_ARG, "rows and cols must be >= 1");
    if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8)) return fail(GPTQ_ERR_INVALID_ARG, "bits must be 2, 3, 4 or 8");
    if (layout != 0 && layout != 1) return fail(GPTQ_ERR_INVALID_ARG, "layout must be 0 or 1");
    const long long words = rows * ((cols * bits + 31) / 32);
    {
        gqh::TimedScope ts__("pack_int", (cudaStream_t)stream);
        gq::pack_int_kernel<<<(unsigned)std::min<long long>((words + 255) / 256, 8192), 256, 0, (cudaStream_t)stream>>>(
            codes, rows, cols, bits, layout, packed);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pack_int");
    return GPTQ_OK;
}

gptq_status gptq_dequant(const int32_t* qweight, const uint16_t* scales, const int32_t* qzeros, int64_t d_out,
                         int64_t d_in, const gptq_config* cfg, float* W_hat, void* stream) {
    return dequant_common(qweight, scales, qzeros, nullptr, d_out, d_in, cfg, W_hat, stream);
}

gptq_status gptq_dequant_g_idx(const int32_t* qweight, const uint16_t* scales, const int32_t* qzeros,
                               const int32_t* g_idx, int64_t d_out, int64_t d_in, const gptq_config* cfg,
                               float* W_hat, void* stream) {
    if (!g_idx) return fail(GPTQ_ERR_INVALID_ARG, "g_idx must be non-NULL");
    return dequant_common(qweight, scales, qzeros, g_idx, d_out, d_in, cfg, W_hat, stream);
}

gptq_status gptq_dequant_gemm(const void* X, int64_t M, const int32_t* qweight, const uint16_t* scales,
                              const int32_t* qzeros, int64_t d_out, int64_t d_in, const gptq_config* cfg, float* Y,
                              void* stream) {
    if (!cfg) return fail(GPTQ_ERR_INVALID_ARG, "cfg is NULL");
    if (!X || !qweight || !scales || !Y) return fail(GPTQ_ERR_INVALID_ARG, "X, qweight, scales and Y must be non-NULL");
    if (cfg->sym ? (qzeros != nullptr) : (qzeros == nullptr))
        return fail(GPTQ_ERR_INVALID_ARG, "qzeros must be given iff asymmetric");
    if (M < 1 || M > (1ll << 30)) return fail(GPTQ_ERR_INVALID_ARG, "M out of range (%lld)", (long long)M);
    if (d_in < 64 || d_in > 65536 || d_in % 64) return fail(GPTQ_ERR_INVALID_ARG, "d_in must be a multiple of 64 in [64, 65536]");
    if (d_out < 8 || d_out > (1ll << 30) || d_out % 8) return fail(GPTQ_ERR_INVALID_ARG, "d_out must be a positive multiple of 8");
    if (!aligned16(X) || !aligned16(qweight) || !aligned16(scales) || !aligned16(Y) || (qzeros && !aligned16(qzeros)))
        return fail(GPTQ_ERR_INVALID_ARG, "X, qweight, scales, qzeros and Y must be 16-byte aligned");
    if (!(cfg->bits == 2 || cfg->bits == 4 || cfg->bits == 8))
        return fail(GPTQ_ERR_UNSUPPORTED, "dequant_gemm: bits must be 2, 4 or 8 (3-bit codes straddle words)");
    const int g = cfg->group_size;
    if (!(g == -1 || (g >= 64 && g % 64 == 0 && d_in % g == 0)))
        return fail(GPTQ_ERR_UNSUPPORTED, "dequant_gemm: group_size must be -1 or a multiple of 64 dividing d_in");
    if (cfg->desc_act) return fail(GPTQ_ERR_UNSUPPORTED, "dequant_gemm: no per-column group index (desc_act)");
    cudaStream_t st = (cudaStream_t)stream;
    const __half* sc = reinterpret_cast<const __half*>(scales);
    cudaError_t e;
    switch (cfg->bits) {
        case 2: e = dq_gemm_run<2>(X, M, qweight, sc, qzeros, d_out, d_in, g, Y, st); break;
        case 4: e = dq_gemm_run<4>(X, M, qweight, sc, qzeros, d_out, d_in, g, Y, st); break;
        default: e = dq_gemm_run<8>(X, M, qweight, sc, qzeros, d_out, d_in, g, Y, st); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "dequant_gemm");
    return GPTQ_OK;
}

size_t gptq_layer_loss_workspace_bytes(int64_t d_out, int64_t d_in, int64_t n) {
    if (d_out < 1 || n < 1 || d_in < 8 || d_out > (1ll << 30) || n > (1ll << 30) || d_in > 65536) return 0;
    return loss_ws_bytes(d_out, d_in, n);
}

gptq_status gptq_layer_loss(const float* W, const float* W_hat, const void* X, gptq_dtype xt, int64_t d_out,
                            int64_t d_in, int64_t n, double* row_loss, double* loss, void* ws, size_t ws_bytes,
                            void* stream) {
    if (!W || !W_hat || !X || !loss) return fail(GPTQ_ERR_INVALID_ARG, "W, W_hat, X and loss must be non-NULL");
    if (xt != GPTQ_BF16 && xt != GPTQ_F32) return fail(GPTQ_ERR_INVALID_ARG, "unknown X dtype %d", (int)xt);
    if (d_out < 1 || d_out > (1ll << 30)) return fail(GPTQ_ERR_INVALID_ARG, "d_out out of range (%lld)", (long long)d_out);
    if (n < 1 || n > (1ll << 30)) return fail(GPTQ_ERR_INVALID_ARG, "n out of range (%lld)", (long long)n);
    if (d_in < 8 || d_in > 65536 || d_in % 8) return fail(GPTQ_ERR_INVALID_ARG, "d_in must be a multiple of 8 in [8, 65536]");
    if (!aligned16(W) || !aligned16(W_hat) || !aligned16(X) || !aligned16(ws) ||
        (reinterpret_cast<uintptr_t>(loss) & 7) || (reinterpret_cast<uintptr_t>(row_loss) & 7))
        return fail(GPTQ_ERR_INVALID_ARG, "W, W_hat, X and ws must be 16-byte aligned, row_loss and loss 8-byte");
    if (!ws || ws_bytes < loss_ws_bytes(d_out, d_in, n))
        return fail(GPTQ_ERR_WORKSPACE, "workspace needs %zu bytes", loss_ws_bytes(d_out, d_in, n));
    cudaError_t e = loss_run(W, W_hat, X, xt == GPTQ_BF16, d_out, d_in, n, row_loss, loss, ws, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "layer_loss");
    return GPTQ_OK;
}

size_t gptq_2d_workspace_bytes(int64_t m, int64_t n, int64_t batch) {
    if (m < 1 || n < 1 || batch < 1) return 0;
    return g2_ws_bytes(m, n, batch);
}

gptq_status gptq_2d_round(const double* X, int64_t m, int64_t n, int64_t batch, const double* U_left,
                          const double* U_right, int32_t* Z, void* ws, size_t ws_bytes, void* stream) {
    if (!X || !U_left || !U_right || !Z) return fail(GPTQ_ERR_INVALID_ARG, "X, U_left, U_right and Z must be non-NULL");
    if (m < 1 || n < 1 || m > 16384 || n > 16384) return fail(GPTQ_ERR_INVALID_ARG, "m and n must be in [1, 16384]");
    if (batch < 1 || batch > (1ll << 20) || batch * m * n > (1ll << 40))
        return fail(GPTQ_ERR_INVALID_ARG, "batch out of range (%lld)", (long long)batch);
    const uintptr_t mis = reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(U_left) |
                          reinterpret_cast<uintptr_t>(U_right) | reinterpret_cast<uintptr_t>(ws);
    if ((mis & 7u) || (reinterpret_cast<uintptr_t>(Z) & 3u))
        return fail(GPTQ_ERR_INVALID_ARG, "X, U_left, U_right and ws must be 8-byte, Z 4-byte aligned");
    const size_t need = g2_ws_bytes(m, n, batch);
    if (!ws || ws_bytes < need) return fail(GPTQ_ERR_WORKSPACE, "workspace needs %zu bytes", need);
    cudaError_t e = g2_run(X, m, n, batch, U_left, U_right, Z, ws, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "gptq_2d_round");
    return GPTQ_OK;
}

gptq_status gptq_sync_status(void* stream) { return read_status((cudaStream_t)stream, nullptr); }

void gptq_timing_enable(int on) { g_timing = on != 0; }

size_t gptq_timing_report(char* buf, size_t len) {
    timing_collect();
    std::string out = "{";
    bool first = true;
    for (auto& kv : g_timing_acc) {
        char item[256];
        snprintf(item, sizeof(item), "%s\"%s\": [%lld, %.6f]", first ? "" : ", ", kv.first.c_str(),
                 kv.second.first, kv.second.second);
        out += item;
        first = false;
    }
    out += "}";
    if (buf && len) {  // a size query (buf == NULL) keeps the totals
        const size_t n = std::min(len - 1, out.size());
        memcpy(buf, out.data(), n);
        buf[n] = 0;
        g_timing_acc.clear();
    }
    return out.size() + 1;
}

size_t gptq_timing_timeline(char* buf, size_t len) {
    timing_collect();
    std::string out = "[";
    for (size_t k = 0; k < g_timeline.size(); ++k) {
        char item[256];
        const TimelineEntry& t = g_timeline[k];
        snprintf(item, sizeof(item), "%s[\"%s\", %d, %.4f, %.4f]", k ? ", " : "", t.name.c_str(), t.stream,
                 (double)t.t0, (double)t.t1);
        out += item;
    }
    out += "]";
    if (buf && len) {
        const size_t n = std::min(len - 1, out.size());
        memcpy(buf, out.data(), n);
        buf[n] = 0;
        g_timeline.clear();
        g_timeline_streams.clear();
    }
    return out.size() + 1;
}

gptq_status gptq_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
    if (limit_ns > 10000000000ull) return fail(GPTQ_ERR_INVALID_ARG, "limit_ns must be <= 10 s");
    {
        TimedScope ts__("selftest_wait", (cudaStream_t)stream);
        gq::selftest_wait_kernel<<<1, 1, 0, (cudaStream_t)stream>>>((unsigned long long)limit_ns);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "selftest_bounded_wait");
    return GPTQ_OK;
}

}  // extern "C"

// ============================================================================
// Fixed-scratch Hessian accumulation (no device or host allocation).
// The scratch for the transposed calibration batch lives in a file-scope device
// array; host code must use its device address, taken with cudaGetSymbolAddress on
// each device the first time this entry point runs there.
// ============================================================================
namespace gq {
constexpr size_t kFixedHessScratchBytes = size_t(16) << 20;
__device__ __align__(256) uint8_t g_fixed_hess_scratch[kFixedHessScratchBytes];
}  // namespace gq

namespace gqh {

constexpr int kMaxDevices = 128;
// Device address of the fixed scratch, looked up once per (device, context): a context that
// was torn down and created again (cudaDeviceReset) may load the module elsewhere.
struct FixedScratchSlot {
    void* ctx;
    void* addr;
};
static FixedScratchSlot g_fixed_scratch_slots[kMaxDevices];   // zero-initialised; one slot per device ordinal

using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
static PfnCtxGetCurrent g_ctx_get_current = nullptr;

static cudaError_t fixed_scratch_address(int dev, void** out) {
    if (!g_ctx_get_current) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return cudaErrorUnknown;
        g_ctx_get_current = reinterpret_cast<PfnCtxGetCurrent>(fn);
    }
    CUcontext ctx = nullptr;   // stays NULL before the runtime has used this device
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
    FixedScratchSlot& slot = g_fixed_scratch_slots[dev];
    if (slot.addr == nullptr || ctx == nullptr || slot.ctx != (void*)ctx) {
        void* addr = nullptr;   // the lookup also initialises the device's primary context
        const cudaError_t e = cudaGetSymbolAddress(&addr, gq::g_fixed_hess_scratch);
        if (e != cudaSuccess) return e;
        if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorUnknown;
        slot.ctx = (void*)ctx;
        slot.addr = addr;
    }
    *out = slot.addr;
    return cudaSuccess;
}

}  // namespace gqh

extern "C" {

gptq_status gptq_hessian_accumulate_fixed_scratch(const void* X, gptq_dtype xt, int64_t n, int64_t d_in, float* H,
                                                  int accumulate, void* stream) {
    if (!X || !H) return fail(GPTQ_ERR_INVALID_ARG, "X and H must be non-NULL");
    if (xt != GPTQ_BF16 && xt != GPTQ_F32) return fail(GPTQ_ERR_INVALID_ARG, "unknown X dtype %d", (int)xt);
    if (n < 1 || n > (1ll << 30)) return fail(GPTQ_ERR_INVALID_ARG, "n out of range (%lld)", (long long)n);
    if (d_in < 8 || d_in > 65536 || d_in % 8) return fail(GPTQ_ERR_INVALID_ARG, "d_in must be a multiple of 8 in [8, 65536]");
    if (!aligned16(X) || !aligned16(H)) return fail(GPTQ_ERR_INVALID_ARG, "X and H must be 16-byte aligned");
    const size_t need = hessian_ws_bytes(n, d_in, xt);
    if (need > gq::kFixedHessScratchBytes)
        return fail(GPTQ_ERR_INVALID_ARG,
                    "batch too large for the fixed scratch: needs %zu bytes, the library holds %zu; "
                    "split the calibration batch or use gptq_hessian_accumulate with a workspace",
                    need, gq::kFixedHessScratchBytes);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(GPTQ_ERR_INVALID_ARG, "device ordinal %d out of range", dev);
    void* ws = nullptr;
    e = fixed_scratch_address(dev, &ws);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(fixed scratch)");
    e = hessian_run(X, xt, n, d_in, H, accumulate ? 1 : 0, ws, (cudaStream_t)stream, true);
    if (e != cudaSuccess) return cuda_fail(e, "fixed-scratch hessian");
    return GPTQ_OK;
}

}  // extern "C"
