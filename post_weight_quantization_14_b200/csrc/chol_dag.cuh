// The blocked factorization of chol.cuh as one persistent dataflow kernel.
//
// With T = n / 128 tiles per side, tile indices i, j, k, m < T, and Hd = R R^T (R upper,
// factored from the bottom-right corner), U = R^-1:
//   LEAF(j)         R_jj from A_jj, X_jj = R_jj^-1                       (one CTA, fp32)
//   PANEL(j, i)     R_ij  = A_ij X_jj^T                      i < j
//   UPDATE(j, i, k) A_ik -= R_ij R_kj^T                       i <= k < j
//   SUPD(i, k, m)   S_im += R_ik U_km                         i < k <= m    (U_mm = X_mm)
//   FIN(i, m)       U_im  = -X_ii S_im                        i < m
// (block back-substitution for U = R^-1: U_im = -X_ii sum_{k=i+1}^{m} R_ik U_km).  Every
// product is one 128 x 128 x 128 tile in 3xTF32 on the tensor cores (tcgen05, operands by
// TMA, accumulators in tensor memory; K split into four segments added in fp32 round-to-
// nearest, cross products apart), with fp32 read-modify-write of A and S in global memory.
//
// One CTA (the first to start) runs the leaves in order j = T-1 .. 0.  Every other CTA
// takes the product tasks from a global ticket counter in a fixed order (dag_step_task):
// per step j the copy of U_jj, the rest of panel j, block column j-1, the far updates, then
// row j of U and the S contributions of panel j.  Each task waits (bounded) for
// the counters of the tasks it reads from, all of which come earlier in that order; so the
// lowest unfinished task can always run, whatever subset of CTAs is resident.  Within a CTA
// the task fetch and TMA loads (warp 0), the MMAs (warp 1) and the epilogue (warps 2-5) are
// pipelined across tasks as in tc_gemm_kernel.  Counters are released by one thread after a
// barrier over the producing threads' stores (gpu-scope fence, then the atomic) and acquired
// before the consuming loads (with a proxy fence in front of TMA reads).
#pragma once
#include "chol.cuh"

namespace gq {

enum : int { DT_PANEL = 0, DT_UPDATE = 1, DT_FIN = 2, DT_SUPD = 3, DT_DIAG = 4, DT_STOP = 15 };

// Optional event trace for profiling builds (GQ_DAG_TRACE defined): %globaltimer stamps of
// each leaf (16 per leaf) and each ticket (8 per ticket, after 16 T leaf slots): fetched,
// inputs ready, first stage landed, accumulator ready, done, CTA.
#ifdef GQ_DAG_TRACE
#define DAG_TRACE(slot, val)                                   \
    do {                                                       \
        if (g_dag_trace) g_dag_trace[(slot)] = (val);          \
    } while (0)
#else
#define DAG_TRACE(slot, val) \
    do {                     \
    } while (0)
#endif

// PANEL(j, i): a = i, b = j.  UPDATE(j, i, k): a = i, b = k, c = j.
// FIN(i, m): a = i, b = m.    SUPD(i, k, m): a = i, b = m, c = k.
// DIAG(j): a = j -- U_jj to the public U and to the U^T split (a copy of X_jj's split).
struct DagTask {
    int type, a, b, c;
    int t;   // ticket (set by the fetching CTA)
};

// Products of step j handed out by ticket.  PANEL(j, j-1) and UPDATE(j, j-1, j-1), the two
// tiles the next leaf needs, are not among them: the leaf CTA forms them itself right after
// LEAF(j) (dag_leaf_role).
__host__ __device__ inline long long dag_step_tasks(int T, int j) {
    const long long jj = j;
    long long c = 1 + (T - 1 - jj) + jj * (T - jj);
    if (j >= 2) c += 2 * (jj - 1) + (jj - 1) * jj / 2;
    return c;
}

__host__ __device__ inline long long dag_total_tasks(int T) {
    long long c = 0;
    for (int j = 0; j < T; ++j) c += dag_step_tasks(T, j);
    return c;
}

// Task idx of step j.
__host__ __device__ inline DagTask dag_step_task(int T, int j, long long idx) {
    if (idx == 0) return DagTask{DT_DIAG, j, 0, 0, 0};
    idx -= 1;
    if (j >= 2) {
        if (idx < j - 1) return DagTask{DT_PANEL, j - 2 - (int)idx, j, 0, 0};
        idx -= j - 1;
        if (idx < j - 1) return DagTask{DT_UPDATE, j - 2 - (int)idx, j - 1, j, 0};
        idx -= j - 1;
        // the far updates, nearest block column first: the next leaves wait for them, so they
        // come before this step's inverse tasks
        for (int k = j - 2; k >= 0; --k) {
            if (idx < k + 1) return DagTask{DT_UPDATE, (int)idx, k, j, 0};
            idx -= k + 1;
        }
    }
    if (idx < T - 1 - j) return DagTask{DT_FIN, j, j + 1 + (int)idx, 0, 0};
    idx -= T - 1 - j;
    if (idx < (long long)j * (T - j)) return DagTask{DT_SUPD, (int)(idx % j), j + (int)(idx / j), j, 0};
    return DagTask{DT_STOP, 0, 0, 0, 0};
}

// Tickets arrive in increasing order per CTA: the cursor walks the steps forward.
struct DagCursor {
    int j;
    long long base;
};
__host__ __device__ inline DagTask dag_decode(int T, DagCursor& cur, long long t) {
    while (cur.j >= 0 && t >= cur.base + dag_step_tasks(T, cur.j)) {
        cur.base += dag_step_tasks(T, cur.j);
        --cur.j;
    }
    if (cur.j < 0) return DagTask{DT_STOP, 0, 0, 0, 0};
    return dag_step_task(T, cur.j, t - cur.base);
}

// Counter block (ints): [0] ticket, [1] role, [2] abort, [3] spare, then T x T arrays
// a_cnt (updates applied to A_ik), rs_done (R_ij final), s_cnt (contributions applied to
// S_im), u_done (U_im final), then leaf_done[T] (X_jj split written) and diag_done[T]
// (U_jj written to U and to the transposed split).
__host__ __device__ inline long long dag_ctr_ints(int T) { return 4 + 4LL * T * T + 2LL * T; }

struct DagArgs {
    int T;
    long long n, d;
    float* A;                    // n x n, damped copy of H (upper tiles), updated in place
    float* S;                    // n x n, S_im accumulators
    float* RS_hi, *RS_lo;        // n x n tf32 split of R (and of the panel inputs)
    float* Xd_hi, *Xd_lo;        // T x 128 x 128 tf32 split of X_jj (row-major)
    float* UT_hi, *UT_lo;        // n x n tf32 split of U^T
    float* TT_hi, *TT_lo;        // n x n tf32 split of S^T
    float* U;                    // d x d public output (strictly lower blocks zeroed beforehand)
    int* ctr;
};

__device__ __forceinline__ int ld_acquire_s32(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ int ld_volatile_s32(const int* p) { return *reinterpret_cast<const volatile int*>(p); }
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Wait until *p >= target.  Bounded: after kWaitLimitNs records GPTQ_ERR_TIMEOUT (with
// `where`) and raises the abort flag; returns false also when another CTA has aborted.
__device__ __noinline__ bool dag_wait_ge(const int* p, int target, int* abort, long long where) {
    if (ld_acquire_s32(p) >= target) return true;
    const unsigned long long t0 = globaltimer_ns();
    unsigned ns = 32;
    for (;;) {
        __nanosleep(ns);
        if (ns < 256) ns <<= 1;
        if (ld_acquire_s32(p) >= target) return true;
        if (ld_volatile_s32(abort)) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_status(GPTQ_ERR_TIMEOUT, where);
            atomicExch(abort, 1);
            return false;
        }
    }
}

// Counters a task waits for (the values it needs are reached exactly when the tasks it
// reads from have completed).
__device__ __forceinline__ bool dag_deps(const DagArgs& g, const DagTask& t) {
    const int T = g.T;
    int* c = g.ctr;
    int* abort = c + 2;
    const int* a_cnt = c + 4;
    const int* rs_done = a_cnt + T * T;
    const int* s_cnt = rs_done + T * T;
    const int* u_done = s_cnt + T * T;
    const int* leaf_done = u_done + T * T;
    const int* diag_done = leaf_done + T;
    const long long where = -(1000000LL + t.type * 100000LL + t.a * 1000LL + t.b);
    switch (t.type) {
        case DT_PANEL:
            return dag_wait_ge(&leaf_done[t.b], 1, abort, where) &&
                   dag_wait_ge(&a_cnt[t.a * T + t.b], T - 1 - t.b, abort, where);
        case DT_UPDATE:
            return dag_wait_ge(&rs_done[t.a * T + t.c], 1, abort, where) &&
                   dag_wait_ge(&rs_done[t.b * T + t.c], 1, abort, where) &&
                   dag_wait_ge(&a_cnt[t.a * T + t.b], T - 1 - t.c, abort, where);
        case DT_FIN:
            return dag_wait_ge(&leaf_done[t.a], 1, abort, where) &&
                   dag_wait_ge(&s_cnt[t.a * T + t.b], t.b - t.a, abort, where);
        case DT_DIAG:
            return dag_wait_ge(&leaf_done[t.a], 1, abort, where);
        case DT_SUPD:
            return dag_wait_ge(&rs_done[t.a * T + t.c], 1, abort, where) &&
                   dag_wait_ge(t.c == t.b ? &diag_done[t.b] : &u_done[t.c * T + t.b], 1, abort, where) &&
                   dag_wait_ge(&s_cnt[t.a * T + t.b], t.b - t.c, abort, where);
    }
    return false;
}

// The counter a completed task advances.
__device__ __forceinline__ int* dag_done_ctr(const DagArgs& g, const DagTask& t) {
    const int T = g.T;
    int* a_cnt = g.ctr + 4;
    int* rs_done = a_cnt + T * T;
    int* s_cnt = rs_done + T * T;
    int* u_done = s_cnt + T * T;
    int* diag_done = u_done + T * T + T;
    switch (t.type) {
        case DT_DIAG: return &diag_done[t.a];
        case DT_PANEL: return &rs_done[t.a * T + t.b];
        case DT_UPDATE: return &a_cnt[t.a * T + t.b];
        case DT_FIN: return &u_done[t.a * T + t.b];
        default: return &s_cnt[t.a * T + t.b];
    }
}

constexpr int DAG_THREADS = 256;                 // the leaf's threads (warps 0-7)
constexpr int DAG_BLOCK = 320;                   // product CTAs: TMA, MMA, 8 epilogue warps
constexpr int DAG_EPI_WARPS = 8;                 // two per TMEM lane quadrant, two chunks each
constexpr int DAG_EPI_BOXES = 3;                 // 32x32 fp32 boxes per epilogue warp: 2 C + 1 staging
constexpr int DAG_STAGES = 2;
constexpr int DAG_SLOTS = 4;
constexpr int DAG_NK = NB / GemmCfg<KIND_TF32X3, 128>::KT;   // 4 TMA stages of K = 32 per task
constexpr int DAG_SEG = 4;                                   // MMA k-steps per accumulator segment
constexpr int DAG_GEMM_BYTES =
    DAG_STAGES * GemmCfg<KIND_TF32X3, 128>::STAGE_BYTES + DAG_EPI_WARPS * DAG_EPI_BOXES * kBoxBytes;

struct DagCtl {
    uint64_t full[DAG_STAGES], empty[DAG_STAGES], tfull[2], tempty[2], cin[DAG_EPI_WARPS];
    uint64_t task_full[DAG_SLOTS], task_empty[DAG_SLOTS];
    DagTask slot[DAG_SLOTS];
    uint32_t tmem_slot;
    int flag;
    int epi_ok[DAG_EPI_WARPS];
};
constexpr int DAG_SMEM_BODY = (DAG_GEMM_BYTES > (int)sizeof(LeafSmem) ? DAG_GEMM_BYTES : (int)sizeof(LeafSmem));
constexpr int DAG_SMEM = 1024 + DAG_SMEM_BODY + (int)sizeof(DagCtl);
static_assert(DAG_SMEM <= 232448, "persistent factorization: shared memory per CTA");
static_assert(NB * NB / 4 == 16 * DAG_THREADS, "leaf load and store loops");

__device__ __forceinline__ void named_bar_epi() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

struct DagMaps {
    // operands (128 x 32 boxes) and C in/out (32 x 32 boxes), all 128-byte swizzled
    CUtensorMap rs_hi, rs_lo, xd_hi, xd_lo, tt_hi, tt_lo, ut_hi, ut_lo, ca, cs;
    // stores of the epilogue (32 x 32 boxes): R's split, U^T's and S^T's splits, the public U
    CUtensorMap rs_hi32, rs_lo32, ut_hi32, ut_lo32, tt_hi32, tt_lo32, u32;
};

// ---------------------------------------------------------------------------------------
// The leaf CTA.  Warps 0-7 (256 threads) form LEAF(j) for j = T-1 .. 0 and, after each leaf
// j >= 1, the two products the next leaf needs, on this CTA's own tensor cores:
//   PANEL(j, j-1):       R_ij = A_ij X_jj^T        (i = j-1; X_jj taken from shared memory)
//   UPDATE(j, j-1, j-1): A_ii - R_ij R_ij^T        (written straight into the next leaf's P)
// R_ij also goes to R's split in global memory (TMA stores) for the other products; U_jj
// goes to the public U and the U^T split by a product task (DIAG(j)).  Warps 8-9 idle.
// Tensor memory (512 columns): three hi*hi segments of 6, 5 and 5 k-steps and the cross
// products apart, summed in fp32 when read; each mbarrier completes once per chain step, so
// its phase parity is the step count.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ int chain_seg(int kk) { return kk < 6 ? 0 : (kk < 11 ? 1 : 2); }
__device__ __forceinline__ bool chain_seg_first(int kk) { return kk == 0 || kk == 6 || kk == 11; }

// One product's 16 k-steps of 3xTF32 MMAs (A rows x K, B rows x K, both K-major, 128-byte
// swizzled; K-slice s of 32 at a_hi(s) / a_lo(s) = a_hi(s) + 16 KB and likewise for B).
template <typename FA, typename FB>
__device__ __forceinline__ void chain_mma_slices(uint32_t tmem, int s0, int s1, FA a_hi, FB b_hi) {
    constexpr uint32_t idesc = make_idesc(2u, BM, 128);
    for (int s = s0; s < s1; ++s) {
        const uint32_t ah = a_hi(s), al = ah + 16384, bh = b_hi(s), bl = bh + 16384;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const int kg = 4 * s + kk;
            const uint32_t off = kk * 32;
            const uint32_t acc = tmem + (uint32_t)(128 * chain_seg(kg));
            umma_tf32(acc, desc_sw128_kmajor(ah + off), desc_sw128_kmajor(bh + off), idesc,
                      chain_seg_first(kg) ? 0u : 1u);
            umma_tf32(tmem + 384u, desc_sw128_kmajor(ah + off), desc_sw128_kmajor(bl + off), idesc, kg > 0 ? 1u : 0u);
            umma_tf32(tmem + 384u, desc_sw128_kmajor(al + off), desc_sw128_kmajor(bh + off), idesc, 1u);
        }
    }
}

// Chunk c (32 columns) of a chain product for this warp's 32 rows: ((s0 + s1) + s2) + x.
__device__ __forceinline__ void chain_fetch(uint32_t tmem, uint32_t lane_off, int c, float (&v)[32]) {
    uint32_t a[32], b[32];
    tmem_ld_32x32b_x32(tmem + (uint32_t)(c * 32) + lane_off, a);
    tmem_ld_32x32b_x32(tmem + (uint32_t)(128 + c * 32) + lane_off, b);
    tmem_ld_wait();
#pragma unroll
    for (int u = 0; u < 32; ++u) v[u] = __uint_as_float(a[u]) + __uint_as_float(b[u]);
    tmem_ld_32x32b_x32(tmem + (uint32_t)(256 + c * 32) + lane_off, a);
    tmem_ld_32x32b_x32(tmem + (uint32_t)(384 + c * 32) + lane_off, b);
    tmem_ld_wait();
#pragma unroll
    for (int u = 0; u < 32; ++u) v[u] = (v[u] + __uint_as_float(a[u])) + __uint_as_float(b[u]);
}

__device__ __forceinline__ void dag_leaf_role(const DagMaps& maps, const DagArgs& g, LeafSmem& S, DagCtl& ctl) {
    const int T = g.T;
    const long long n = g.n;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int* c = g.ctr;
    int* abort = c + 2;
    int* a_cnt = c + 4;
    int* rs_done = a_cnt + T * T;
    int* leaf_done = a_cnt + 4 * T * T;
    uint8_t* buf0 = reinterpret_cast<uint8_t*>(&S.P[0][0]);    // chain operand slices 0, 1
    uint8_t* buf1 = reinterpret_cast<uint8_t*>(&S.LT[0][0]);   // chain operand slices 2, 3
    uint8_t* cbuf = reinterpret_cast<uint8_t*>(&S.X[0][0]);    // A_ii, 16 boxes of 32 x 32
    // barriers, one completion per chain step each: A slices 0-3 landed (full[0], full[1],
    // empty[0], empty[1]), slices 0-1 consumed (tempty[0]), panel done (tfull[0]), update
    // done (tfull[1]), A_ii landed (cin[0])
    uint64_t* bar_a[4] = {&ctl.full[0], &ctl.full[1], &ctl.empty[0], &ctl.empty[1]};
    if (tid == 0) {
        for (int q = 0; q < 4; ++q) mbar_init(bar_a[q], 1);
        mbar_init(&ctl.tempty[0], 1);
        mbar_init(&ctl.tfull[0], 1);
        mbar_init(&ctl.tfull[1], 1);
        mbar_init(&ctl.cin[0], 1);
        fence_mbar_init();
        ctl.flag = 1;
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(&ctl.tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_slot;

    if (warp == DAG_THREADS / 32) {
        // ---- warp 8: per chain step j >= 1, X_jj's split (the panel tile's B slices) to global
        // memory, then leaf_done; R_ij (the panel tile) to R's split, then rs_done; three
        // handshakes with warps 0-7 (barrier 6: slices written, barrier 7: slices read by the TMA)
        for (int j = T - 1; j >= 1; --j) {
            const int i = j - 1, ib = i * NB;
            int* leaf_done_ = a_cnt + 4 * T * T;
            // X slices s0, s0 + 1: B hi at buffer + 32 KB, lo at + 48 KB, 128 rows x 32 columns each
            auto store_x = [&](int s0) {
                for (int sl = s0; sl < s0 + 2; ++sl) {
                    uint8_t* bh = ((sl & 1) ? buf1 : buf0) + 32768;
                    tma_store_2d(&maps.xd_hi, bh, 32 * sl, j * NB);
                    tma_store_2d(&maps.xd_lo, bh + 16384, 32 * sl, j * NB);
                }
                bulk_commit();
                bulk_wait_read<0>();
            };
            for (int hs = 0; hs < 2; ++hs) {   // X_jj's split, two slices at a time
                nbar_sync(6, DAG_THREADS + 32);
                const bool st = ctl.flag != 0;
                if (lane == 0 && st) store_x(2 * hs);
                __syncwarp();
                nbar_arrive(7, DAG_THREADS + 32);
            }
            if (lane == 0 && ctl.flag) {
                bulk_wait<0>();
                fence_proxy_async_global();
                __threadfence();
                atomicAdd(&leaf_done_[j], 1);
                DAG_TRACE(16 * j + 1, globaltimer_ns());
            }
            __syncwarp();
            nbar_sync(6, DAG_THREADS + 32);   // R_ij's slices
            const bool st = ctl.flag != 0;
            if (lane == 0 && st) {
                for (int cc = 0; cc < 4; ++cc)
                    for (int qq = 0; qq < 4; ++qq) {
                        uint8_t* sh = ((cc >> 1) ? buf1 : buf0) + (cc & 1) * 32768 + qq * 4096;
                        tma_store_2d(&maps.rs_hi32, sh, j * NB + 32 * cc, ib + 32 * qq);
                        tma_store_2d(&maps.rs_lo32, sh + 16384, j * NB + 32 * cc, ib + 32 * qq);
                    }
                bulk_commit();
                bulk_wait_read<0>();
            }
            __syncwarp();
            nbar_arrive(7, DAG_THREADS + 32);
            if (lane == 0 && st) {
                bulk_wait<0>();
                fence_proxy_async_global();
                __threadfence();
                atomicAdd(&rs_done[i * T + j], 1);
                DAG_TRACE(16 * j + 8, globaltimer_ns());
            }
            __syncwarp();
        }
    } else if (warp < DAG_THREADS / 32) {   // warp 9 takes no part
        // ---- warps 0-7: the leaves and the chain products
        const int q = warp & 3, h = warp >> 2;              // TMEM lane quadrant, chunk half
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        bool have_tile = false;   // P already holds the next leaf's tile (from the chain step)
        for (int j = T - 1; j >= 0; --j) {
            const long long jb = (long long)j * NB;
            const uint32_t par = (uint32_t)((T - 1 - j) & 1);   // chain step count parity
            // ctl.flag is written by thread 0 only between barriers; every branch that holds a
            // barrier takes its condition from a value all threads read after the same barrier
            const bool need_load = ctl.flag && !have_tile;
            leaf_sync();
            if (need_load) {
                if (tid == 0) {
                    if (!dag_wait_ge(&a_cnt[j * T + j], T - 1 - j, abort, -(2000000LL + j))) ctl.flag = 0;
                    DAG_TRACE(16 * j, globaltimer_ns());
                }
                leaf_sync();
                if (ctl.flag) {   // P[127-r][127-c] = A[r][c]
#pragma unroll
                    for (int quarter = 0; quarter < 4; ++quarter) {
                        float4 v[4];
#pragma unroll
                        for (int it = 0; it < 4; ++it) {
                            const int e = tid + (4 * quarter + it) * DAG_THREADS, r = e >> 5, cc = (e & 31) * 4;
                            v[it] = __ldcg(reinterpret_cast<const float4*>(g.A + (jb + r) * n + jb + cc));
                        }
#pragma unroll
                        for (int it = 0; it < 4; ++it) {
                            const int e = tid + (4 * quarter + it) * DAG_THREADS, r = e >> 5, cc = (e & 31) * 4;
                            S.P[127 - r][127 - cc] = v[it].x;
                            S.P[127 - r][126 - cc] = v[it].y;
                            S.P[127 - r][125 - cc] = v[it].z;
                            S.P[127 - r][124 - cc] = v[it].w;
                        }
                    }
                }
                leaf_sync();
            } else if (tid == 0) {
                DAG_TRACE(16 * j, globaltimer_ns());
            }
            const bool alive = ctl.flag != 0;
            const bool chain = alive && j >= 1;
            const int i = j - 1;
            const int ib = i * NB;
            // chain operand slice s (K = 32 s .. 32 s + 31): slices 0, 1 in buf0 / buf1, then
            // 2, 3 again; [A hi | A lo | B hi | B lo], 16 KB each
            auto slice_buf = [&](int s) { return (s & 1) ? buf1 : buf0; };
            // B slices of the panel: X_jj rows n, columns 32 s .. (U_jj[n][k] = S.X[127-n][127-k])
            auto put_x_slices = [&](int s0) {
                for (int sl = s0; sl < s0 + 2; ++sl) {
                    uint8_t* bh = slice_buf(sl) + 32768;
                    const int nrow = tid >> 1, c4b = (tid & 1) * 4;
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const int c4 = c4b + e4, k = 32 * sl + 4 * c4;
                        const float4 xv = ld4(&S.X[127 - nrow][124 - k]);
                        float v[4] = {xv.w, xv.z, xv.y, xv.x};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (nrow > k + e) v[e] = 0.f;
                        float hh[4], ll[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            hh[e] = to_tf32(v[e]);
                            ll[e] = v[e] - hh[e];
                        }
                        const uint32_t off = (uint32_t)(nrow * 128 + ((c4 ^ (nrow & 7)) << 4));
                        *reinterpret_cast<float4*>(bh + off) = make_float4(hh[0], hh[1], hh[2], hh[3]);
                        *reinterpret_cast<float4*>(bh + 16384 + off) = make_float4(ll[0], ll[1], ll[2], ll[3]);
                    }
                }
            };
            auto load_a_slices = [&](int s0) {   // tid 0: A_ij's split, slices s0, s0 + 1
                for (int sl = s0; sl < s0 + 2; ++sl) {
                    uint8_t* ab = slice_buf(sl);
                    mbar_arrive_expect_tx(bar_a[sl], 32768);
                    tma_load_2d(ab, &maps.rs_hi, bar_a[sl], (int)jb + 32 * sl, ib);
                    tma_load_2d(ab + 16384, &maps.rs_lo, bar_a[sl], (int)jb + 32 * sl, ib);
                }
            };
            auto panel_a = [&](int s) { return smem_u32(slice_buf(s)); };
            auto panel_b = [&](int s) { return smem_u32(slice_buf(s)) + 32768u; };
            bool ok = true;
            if (alive) {
                if (tid == 0) DAG_TRACE(16 * j + 12, globaltimer_ns());
                leaf_factor(S, (int)jb);
            }
            have_tile = false;
            if (!chain) {
                if (alive) {   // the last leaf: X_jj's split stored by the leaf warps
                    float* xh = g.Xd_hi + (long long)j * NB * NB;
                    float* xl = g.Xd_lo + (long long)j * NB * NB;
#pragma unroll 4
                    for (int it = 0; it < 16; ++it) {
                        const int task = tid + it * DAG_THREADS, r = task >> 5, cc = (task & 31) * 4;
                        const float4 xv = ld4(&S.X[127 - r][124 - cc]);
                        float v[4] = {xv.w, xv.z, xv.y, xv.x};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (r > cc + e) v[e] = 0.f;
                        float hh[4], ll[4];   // lo unrounded: hi + lo restores X_jj exactly
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            hh[e] = to_tf32(v[e]);
                            ll[e] = v[e] - hh[e];
                        }
                        *reinterpret_cast<float4*>(xh + r * NB + cc) = make_float4(hh[0], hh[1], hh[2], hh[3]);
                        *reinterpret_cast<float4*>(xl + r * NB + cc) = make_float4(ll[0], ll[1], ll[2], ll[3]);
                    }
                    leaf_sync();
                    if (tid == 0) {   // release: the stores (ordered by the barrier), then the counter
                        fence_proxy_async_global();
                        __threadfence();
                        atomicAdd(&leaf_done[j], 1);
                        DAG_TRACE(16 * j + 1, globaltimer_ns());
                    }
                }
                if (j >= 1)   // keep the store warp's three handshakes (see below) in step
                    for (int hs = 0; hs < 3; ++hs) {
                        nbar_arrive(6, DAG_THREADS + 32);
                        nbar_sync(7, DAG_THREADS + 32);
                    }
                continue;
            }

            // ---------------- the chain products of step j (i = j - 1).  X_jj's split is formed
            // once, as the panel tile's B operand; warp 8 stores those slices to X_jj's split in
            // global memory (then leaf_done) and, later, R_ij's slices (then rs_done), while
            // these warps go on; each store is a handshake (barrier 6: written, 7: read).
            if (tid == 0) {
                ok = dag_wait_ge(&a_cnt[i * T + j], T - 1 - j, abort, -(2200000LL + j));
                if (ok) {
                    fence_proxy_async_global();
                    load_a_slices(0);
                } else {
                    ctl.flag = 0;
                }
            }
            put_x_slices(0);
            fence_proxy_async_smem();
            leaf_sync();
            nbar_arrive(6, DAG_THREADS + 32);   // X slices 0-1 written
            if (tid == 0 && ok) {
                DAG_TRACE(16 * j + 3, globaltimer_ns());
                for (int sl = 0; sl < 2 && ok; ++sl) {
                    ok = mbar_wait(bar_a[sl], par, -(2300000LL + j));
                    tc_fence_after();
                    if (ok) chain_mma_slices(tmem, sl, sl + 1, panel_a, panel_b);
                }
                umma_commit(&ctl.tempty[0]);
                ok = ok && mbar_wait(&ctl.tempty[0], par, -(2400000LL + j));   // slices 0-1 consumed
                if (ok) load_a_slices(2);
                if (!ok) ctl.flag = 0;
            }
            nbar_sync(7, DAG_THREADS + 32);     // ... and read by the TMA
            if (tid == 0) DAG_TRACE(16 * j + 4, globaltimer_ns());
            if (ctl.flag) put_x_slices(2);
            fence_proxy_async_smem();
            leaf_sync();
            nbar_arrive(6, DAG_THREADS + 32);   // X slices 2-3 written
            if (tid == 0 && ctl.flag) {
                for (int sl = 2; sl < 4 && ok; ++sl) {
                    ok = mbar_wait(bar_a[sl], par, -(2300000LL + j));
                    tc_fence_after();
                    if (ok) chain_mma_slices(tmem, sl, sl + 1, panel_a, panel_b);
                }
                umma_commit(&ctl.tfull[0]);
                if (!ok) ctl.flag = 0;
            }
            // A_ii (its other updates done) into S.X's space (X_jj is no longer read)
            if (tid == 0 && ctl.flag) {
                if (dag_wait_ge(&a_cnt[i * T + i], T - 1 - j, abort, -(2500000LL + j))) {
                    fence_proxy_async_global();
                    mbar_arrive_expect_tx(&ctl.cin[0], NB * NB * 4);
                    for (int b = 0; b < 16; ++b)
                        tma_load_2d(cbuf + b * 4096, &maps.ca, &ctl.cin[0], ib + 32 * (b & 3), ib + 32 * (b >> 2));
                } else {
                    ctl.flag = 0;
                }
            }
            // R_ij: from tensor memory to the update's operand slices (both A and B); warp
            // (q, h) takes rows 32q.., chunks 2h, 2h+1.  Warp 8 stores the slices to R's split
            // in global memory by TMA and releases rs_done, off this chain.
            bool wok = mbar_wait(&ctl.tfull[0], par, -(2600000LL + j));
            tc_fence_after();
            nbar_sync(7, DAG_THREADS + 32);     // X slices 2-3 read by the TMA
            if (tid == 0) DAG_TRACE(16 * j + 5, globaltimer_ns());
            if (wok) {
                for (int cl = 0; cl < 2; ++cl) {
                    const int cc = 2 * h + cl;
                    float v[32];
                    chain_fetch(tmem, lane_off, cc, v);
                    float hh[32], ll[32];
#pragma unroll
                    for (int u = 0; u < 32; ++u) split_tf32(v[u], hh[u], ll[u]);
                    uint8_t* sh = ((cc >> 1) ? buf1 : buf0) + (cc & 1) * 32768 + q * 4096;   // rows 32q.. of slice cc
                    box_put_row(sh, lane, hh);
                    box_put_row(sh + 16384, lane, ll);
                }
            } else if (lane == 0) {
                ctl.flag = 0;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            nbar_arrive(6, DAG_THREADS + 32);   // the slices are written: warp 8 may store them
            leaf_sync();
            if (tid == 0 && ctl.flag) {   // the update: A = B = R_ij's slices (cc: buffer cc >> 1, half cc & 1)
                DAG_TRACE(16 * j + 6, globaltimer_ns());
                tc_fence_after();
                auto upd = [&](int cc) { return smem_u32((cc >> 1) ? buf1 : buf0) + (uint32_t)((cc & 1) * 32768); };
                chain_mma_slices(tmem, 0, 4, upd, upd);
                umma_commit(&ctl.tfull[1]);
            }
            // the next leaf's tile: P[127-r][127-c] = A_ii[r][c] - (R R^T)[r][c]
            wok = ctl.flag && mbar_wait(&ctl.tfull[1], par, -(2700000LL + j)) &&
                  mbar_wait(&ctl.cin[0], par, -(2800000LL + j));
            tc_fence_after();
            nbar_sync(7, DAG_THREADS + 32);   // warp 8's stores have read the slices P overlays
            if (tid == 0) DAG_TRACE(16 * j + 7, globaltimer_ns());
            if (wok) {
                for (int cl = 0; cl < 2; ++cl) {
                    const int cc = 2 * h + cl;
                    float v[32];
                    chain_fetch(tmem, lane_off, cc, v);
                    const uint8_t* cb = cbuf + (q * 4 + cc) * 4096;   // box (rows 32q.., columns 32 cc..)
                    const int r = 32 * q + lane;
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 a4 = *reinterpret_cast<const float4*>(cb + lane * 128 + ((c4 ^ (lane & 7)) << 4));
                        const int col = 32 * cc + 4 * c4;
                        S.P[127 - r][127 - col] = a4.x - v[4 * c4 + 0];
                        S.P[127 - r][126 - col] = a4.y - v[4 * c4 + 1];
                        S.P[127 - r][125 - col] = a4.z - v[4 * c4 + 2];
                        S.P[127 - r][124 - col] = a4.w - v[4 * c4 + 3];
                    }
                }
            } else if (lane == 0) {
                ctl.flag = 0;
            }
            tc_fence_before();
            leaf_sync();
            have_tile = ctl.flag != 0;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------------------
// Product CTAs.
// ---------------------------------------------------------------------------------------

__global__ void __launch_bounds__(DAG_BLOCK, 1)
    chol_dag_kernel(const __grid_constant__ DagMaps maps, const DagArgs g) {
    extern __shared__ uint8_t dag_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dag_raw) + 1023) & ~uintptr_t(1023));
    DagCtl& ctl = *reinterpret_cast<DagCtl*>(smem + DAG_SMEM_BODY);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = g.T;
    int* abort = g.ctr + 2;

    if (threadIdx.x == 0) ctl.flag = atomicAdd(g.ctr + 1, 1);
    __syncthreads();
    if (ctl.flag == 0) {   // the first CTA to start runs the leaves
        __syncthreads();
        dag_leaf_role(maps, g, *reinterpret_cast<LeafSmem*>(smem), ctl);
        return;
    }

    using Cfg = GemmCfg<KIND_TF32X3, 128>;
    constexpr int TBN = 128, KT = Cfg::KT, STAGE_BYTES = Cfg::STAGE_BYTES;
    constexpr int A_BYTES = BM * 128, B_BYTES = TBN * 128;
    constexpr int SUM_HI = 2 * TBN, XOFF = 3 * TBN;
    constexpr uint32_t TMEM_COLS = 512;
    uint8_t* epi = smem + DAG_STAGES * STAGE_BYTES;

    if (threadIdx.x == 0) {
        for (int s = 0; s < DAG_STAGES; ++s) {
            mbar_init(&ctl.full[s], 1);
            mbar_init(&ctl.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl.tfull[b], 1);
            mbar_init(&ctl.tempty[b], DAG_EPI_WARPS);
        }
        for (int q = 0; q < DAG_EPI_WARPS; ++q) mbar_init(&ctl.cin[q], 1);
        for (int s = 0; s < DAG_SLOTS; ++s) {
            mbar_init(&ctl.task_full[s], 1);
            mbar_init(&ctl.task_empty[s], 1);
        }
        fence_mbar_init();
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(&ctl.tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_slot;

    if (warp == 0 && lane == 0) {
        // ---------------- task fetch, dependency waits, TMA producer
        prefetch_tmap(&maps.rs_hi);
        prefetch_tmap(&maps.rs_lo);
        prefetch_tmap(&maps.xd_hi);
        prefetch_tmap(&maps.xd_lo);
        prefetch_tmap(&maps.tt_hi);
        prefetch_tmap(&maps.tt_lo);
        prefetch_tmap(&maps.ut_hi);
        prefetch_tmap(&maps.ut_lo);
        DagCursor cur{T - 1, 0};
        uint32_t kiter = 0;
        for (int nt = 0;; ++nt) {
            const int s = nt % DAG_SLOTS;
            DagTask tk{DT_STOP, 0, 0, 0};
            const bool slot_ok = mbar_wait(&ctl.task_empty[s], (uint32_t)((nt / DAG_SLOTS) & 1) ^ 1u, -3000000LL - blockIdx.x);
            if (slot_ok && !ld_volatile_s32(abort)) {
                const long long t = atomicAdd(g.ctr, 1);
                DAG_TRACE(16 * T + 8 * t + 0, globaltimer_ns());
                tk = dag_decode(T, cur, t);
                if (tk.type != DT_STOP && !dag_deps(g, tk)) tk.type = DT_STOP;
                if (tk.type != DT_STOP) {
                    DAG_TRACE(16 * T + 8 * t + 1, globaltimer_ns());
                    DAG_TRACE(16 * T + 8 * t + 5, blockIdx.x);
                    tk.t = (int)t;
                }
            } else if (!slot_ok) {
                atomicExch(abort, 1);
            }
            ctl.slot[s] = tk;
            mbar_arrive(&ctl.task_full[s]);
            if (tk.type == DT_STOP) break;
            if (tk.type == DT_DIAG) continue;   // no operands: the epilogue warps copy
            fence_proxy_async_global();   // the counters were acquired; TMA reads follow
            const CUtensorMap *ma_h, *ma_l, *mb_h, *mb_l;
            int ax, ay, bx, by;
            switch (tk.type) {
                case DT_PANEL:   // A = R-split(i, j) (the updated panel input), B = X_jj
                    ma_h = &maps.rs_hi; ma_l = &maps.rs_lo; ax = tk.b * NB; ay = tk.a * NB;
                    mb_h = &maps.xd_hi; mb_l = &maps.xd_lo; bx = 0; by = tk.b * NB;
                    break;
                case DT_UPDATE:  // A = R(i, j), B = R(k, j)
                    ma_h = &maps.rs_hi; ma_l = &maps.rs_lo; ax = tk.c * NB; ay = tk.a * NB;
                    mb_h = &maps.rs_hi; mb_l = &maps.rs_lo; bx = tk.c * NB; by = tk.b * NB;
                    break;
                case DT_FIN:     // A = X_ii, B = S_im^T
                    ma_h = &maps.xd_hi; ma_l = &maps.xd_lo; ax = 0; ay = tk.a * NB;
                    mb_h = &maps.tt_hi; mb_l = &maps.tt_lo; bx = tk.a * NB; by = tk.b * NB;
                    break;
                default:         // SUPD: A = R(i, k), B = U_km^T
                    ma_h = &maps.rs_hi; ma_l = &maps.rs_lo; ax = tk.c * NB; ay = tk.a * NB;
                    mb_h = &maps.ut_hi; mb_l = &maps.ut_lo; bx = tk.c * NB; by = tk.b * NB;
                    break;
            }
            for (int kt = 0; kt < DAG_NK; ++kt, ++kiter) {
                const int st = kiter % DAG_STAGES;
                const uint32_t it = kiter / DAG_STAGES;
                if (!mbar_wait(&ctl.empty[st], (it & 1) ^ 1, -4000000LL - blockIdx.x)) {
                    atomicExch(abort, 1);
                    break;
                }
                uint8_t* sb = smem + st * STAGE_BYTES;
                mbar_arrive_expect_tx(&ctl.full[st], STAGE_BYTES);
                const int k = kt * KT;
                tma_load_2d(sb, ma_h, &ctl.full[st], ax + k, ay);
                tma_load_2d(sb + A_BYTES, ma_l, &ctl.full[st], ax + k, ay);
                tma_load_2d(sb + 2 * A_BYTES, mb_h, &ctl.full[st], bx + k, by);
                tma_load_2d(sb + 2 * A_BYTES + B_BYTES, mb_l, &ctl.full[st], bx + k, by);
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer (segmented accumulation as in tc_gemm_kernel)
        constexpr uint32_t idesc = make_idesc(2u, BM, TBN);
        const uint32_t xacc = tmem + (uint32_t)XOFF;
        uint32_t kiter = 0;
        int seg = 0;
        bool ok = true;
        for (int nt = 0; ok; ++nt) {
            const int s = nt % DAG_SLOTS;
            if (!mbar_wait(&ctl.task_full[s], (uint32_t)(nt / DAG_SLOTS) & 1, -5000000LL - blockIdx.x)) break;
            const DagTask tk = ctl.slot[s];
            if (tk.type == DT_STOP) break;
            if (tk.type == DT_DIAG) continue;
            if (seg > 0) {   // the previous task's cross accumulator has been read
                const int pb = (seg - 1) & 1;
                if (!mbar_wait(&ctl.tempty[pb], (uint32_t)((seg - 1) >> 1) & 1, -5100000LL - blockIdx.x)) break;
                tc_fence_after();
            }
            auto open_segment = [&](uint32_t& acc_out) -> bool {
                const int buf = seg & 1;
                if (!mbar_wait(&ctl.tempty[buf], (uint32_t)((seg >> 1) & 1) ^ 1u, -5200000LL - blockIdx.x))
                    return false;
                tc_fence_after();
                acc_out = tmem + (uint32_t)(buf * TBN);
                return true;
            };
            uint32_t acc = 0;
            if (!open_segment(acc)) break;
            int kkc = 0, segpos = 0;
            for (int kt = 0; kt < DAG_NK && ok; ++kt, ++kiter) {
                const int st = kiter % DAG_STAGES;
                const uint32_t it = kiter / DAG_STAGES;
                if (!mbar_wait(&ctl.full[st], it & 1, -5300000LL - blockIdx.x)) {
                    ok = false;
                    break;
                }
                if (kt == 0) DAG_TRACE(16 * T + 8 * (long long)tk.t + 2, globaltimer_ns());
                tc_fence_after();
                const uint32_t sb = smem_u32(smem + st * STAGE_BYTES);
                const uint32_t a_hi = sb, a_lo = sb + A_BYTES;
                const uint32_t b_hi = sb + 2 * A_BYTES, b_lo = b_hi + B_BYTES;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk, ++kkc, ++segpos) {
                    if (segpos == DAG_SEG) {
                        umma_commit(&ctl.tfull[seg & 1]);
                        ++seg;
                        segpos = 0;
                        if (!open_segment(acc)) {
                            ok = false;
                            break;
                        }
                    }
                    const uint32_t off = kk * 32;
                    const uint32_t acc0 = segpos > 0 ? 1u : 0u;
                    const uint32_t x0 = kkc > 0 ? 1u : 0u;
                    umma_tf32(acc, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_hi + off), idesc, acc0);
                    umma_tf32(xacc, desc_sw128_kmajor(a_hi + off), desc_sw128_kmajor(b_lo + off), idesc, x0);
                    umma_tf32(xacc, desc_sw128_kmajor(a_lo + off), desc_sw128_kmajor(b_hi + off), idesc, 1u);
                }
                umma_commit(&ctl.empty[st]);
            }
            if (!ok) break;
            umma_commit(&ctl.tfull[seg & 1]);
            ++seg;
        }
    } else if (warp >= 2) {
        // ---------------- epilogue: warp w (2..9) owns accumulator rows 32q .. 32q+31, q = w % 4,
        // and the chunks (32 columns each) 2h, 2h+1 of them, h = (w - 2) / 4
        const int q = warp & 3, ew = warp - 2, h = ew >> 2;
        uint8_t* wreg = epi + ew * DAG_EPI_BOXES * kBoxBytes;
        uint8_t* cbox = wreg;                      // this warp's two C chunks
        uint8_t* kb = wreg + 2 * kBoxBytes;        // staging box
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        constexpr int nseg = DAG_NK * 4 / DAG_SEG;
        int seg = 0;
        uint32_t cin_use = 0;
        for (int nt = 0;; ++nt) {
            const int s = nt % DAG_SLOTS;
            // the four warps agree on whether a task came (each wait is bounded), so none of
            // them can be left alone at the task's named barriers
            const bool got = mbar_wait(&ctl.task_full[s], (uint32_t)(nt / DAG_SLOTS) & 1, -6000000LL - blockIdx.x);
            if (lane == 0) ctl.epi_ok[ew] = got ? 1 : 0;
            named_bar_epi();
            bool all = true;
#pragma unroll
            for (int e = 0; e < DAG_EPI_WARPS; ++e) all = all && ctl.epi_ok[e];
            const DagTask tk = ctl.slot[s];
            named_bar_epi();
            if (!all || tk.type == DT_STOP) break;
            if (tk.type == DT_DIAG) {
                // U_jj = X_jj hi + lo (exact: lo is unrounded) to the public U (clipped), and
                // the split transposed to U^T: 32 x 32 blocks through this warp's staging box
                const long long jb = (long long)tk.a * NB, nn = g.n;
                const float* xh = g.Xd_hi + (long long)tk.a * NB * NB;
                const float* xl = g.Xd_lo + (long long)tk.a * NB * NB;
                for (int bk = ew; bk < 16; bk += DAG_EPI_WARPS) {
                    const int bi = bk >> 2, bj = bk & 3;
                    float vh[32], vl[32], vu[32];
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 a4 = __ldcg(reinterpret_cast<const float4*>(xh + (32 * bi + lane) * NB + 32 * bj + 4 * c4));
                        const float4 b4 = __ldcg(reinterpret_cast<const float4*>(xl + (32 * bi + lane) * NB + 32 * bj + 4 * c4));
                        vh[4 * c4] = a4.x, vh[4 * c4 + 1] = a4.y, vh[4 * c4 + 2] = a4.z, vh[4 * c4 + 3] = a4.w;
                        vl[4 * c4] = b4.x, vl[4 * c4 + 1] = b4.y, vl[4 * c4 + 2] = b4.z, vl[4 * c4 + 3] = b4.w;
                    }
#pragma unroll
                    for (int u = 0; u < 32; ++u) vu[u] = vh[u] + vl[u];
                    emit_block(kb, lane, vu, false, g.U, g.d, g.d, g.d, jb + 32 * bi, jb + 32 * bj);
                    emit_block(kb, lane, vh, true, g.UT_hi, nn, nn, nn, jb + 32 * bj, jb + 32 * bi);
                    emit_block(kb, lane, vl, true, g.UT_lo, nn, nn, nn, jb + 32 * bj, jb + 32 * bi);
                }
                named_bar_epi();
                if (warp == 2 && lane == 0) {
                    fence_proxy_async_global();
                    __threadfence();
                    atomicAdd(dag_done_ctr(g, tk), 1);
                    DAG_TRACE(16 * (long long)tk.a + 2, globaltimer_ns());
                    mbar_arrive(&ctl.task_empty[s]);
                }
                continue;
            }
            // the task's epilogue: outputs
            const long long n = g.n;
            const int i0 = tk.a * NB + 32 * q;   // first tile row of this warp (global row)
            float alpha = 1.f, beta = 0.f;
            bool C = false;
            long long c_rows = n, c_cols = n, c_col0 = 0;
            const CUtensorMap* mc = nullptr;         // C load
            const CUtensorMap* mc_store = nullptr;   // C store
            bool s_split = false;
            const CUtensorMap *t_hi = nullptr, *t_lo = nullptr;
            long long t_row0 = 0;
            long long s_col0 = 0;
            switch (tk.type) {
                case DT_PANEL:
                    s_split = true;
                    s_col0 = (long long)tk.b * NB;
                    break;
                case DT_UPDATE:
                    alpha = -1.f;
                    beta = 1.f;
                    C = true;
                    mc = mc_store = &maps.ca;
                    c_col0 = (long long)tk.b * NB;
                    s_split = (tk.b == tk.c - 1) && (tk.a < tk.b);   // the next panel's input
                    s_col0 = c_col0;
                    break;
                case DT_FIN:
                    alpha = -1.f;
                    C = true;
                    mc_store = &maps.u32;
                    c_rows = g.d;
                    c_cols = g.d;
                    c_col0 = (long long)tk.b * NB;
                    t_hi = &maps.ut_hi32;
                    t_lo = &maps.ut_lo32;
                    t_row0 = (long long)tk.b * NB;
                    break;
                default:   // SUPD
                    beta = (tk.c == tk.b) ? 0.f : 1.f;
                    C = true;
                    mc = mc_store = &maps.cs;
                    c_col0 = (long long)tk.b * NB;
                    if (tk.c == tk.a + 1) {
                        t_hi = &maps.tt_hi32;
                        t_lo = &maps.tt_lo32;
                        t_row0 = (long long)tk.b * NB;
                    }
                    break;
            }
            // C (beta != 0) is fetched now, while the MMAs run
            if (beta != 0.f) {
                fence_proxy_async_smem();   // this warp's reads of cbox (previous task) come first
                __syncwarp();
                if (lane == 0) {
                    fence_proxy_async_global();   // C was written by another task (acquired by warp 0)
                    mbar_arrive_expect_tx(&ctl.cin[ew], 2 * kBoxBytes);
                    for (int cl = 0; cl < 2; ++cl)
                        tma_load_2d(cbox + cl * kBoxBytes, mc, &ctl.cin[ew], (int)(c_col0 + 32 * (2 * h + cl)), i0);
                }
                __syncwarp();
            }
            bool ok = true;
            // segments before the last: add into the running sum (columns SUM_HI ..)
            for (int sg = 0; sg + 1 < nseg && ok; ++sg, ++seg) {
                const int sb = seg & 1;
                ok = mbar_wait(&ctl.tfull[sb], (uint32_t)(seg >> 1) & 1, -6100000LL - blockIdx.x);
                tc_fence_after();
#pragma unroll 1
                for (int c = 2 * h; c < 2 * h + 2; ++c) {
                    const uint32_t src = tmem + (uint32_t)(sb * TBN + c * 32) + lane_off;
                    const uint32_t dhi = tmem + (uint32_t)(SUM_HI + c * 32) + lane_off;
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(src, r);
                    if (sg > 0) {
                        uint32_t t[32];
                        tmem_ld_32x32b_x32(dhi, t);
                        tmem_ld_wait();
#pragma unroll
                        for (int u = 0; u < 32; ++u)
                            r[u] = __float_as_uint(__uint_as_float(r[u]) + __uint_as_float(t[u]));
                    } else {
                        tmem_ld_wait();
                    }
                    tmem_st_32x32b_x32(dhi, r);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.tempty[sb]);
            }
            const int buf = seg & 1;
            const uint32_t use = (uint32_t)(seg >> 1);
            ++seg;
            ok = ok && mbar_wait(&ctl.tfull[buf], use & 1, -6200000LL - blockIdx.x);
            if (warp == 2 && lane == 0) DAG_TRACE(16 * T + 8 * (long long)tk.t + 3, globaltimer_ns());
            tc_fence_after();
            const uint32_t acc = tmem + (uint32_t)(buf * TBN) + lane_off;

            bool cin_ok = true;
            if (beta != 0.f) {
                cin_ok = mbar_wait(&ctl.cin[ew], cin_use & 1, -6300000LL - blockIdx.x);
                ++cin_use;
                if (warp == 2 && lane == 0) DAG_TRACE(16 * T + 8 * (long long)tk.t + 7, globaltimer_ns());
            }
#pragma unroll 1
            for (int cl = 0; cl < 2; ++cl) {
                const int c = 2 * h + cl;   // chunk: columns 32c .. 32c+31 of the tile
                uint32_t r[32];
                if (ok) {
                    fetch_chunk<TBN, true, false>(tmem, acc, lane_off, c, true, r);
                } else {
#pragma unroll
                    for (int u = 0; u < 32; ++u) r[u] = 0u;
                }
                if (cl == 1) {   // this warp has read its part of the accumulator
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ctl.tempty[buf]);
                }
                float out[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) out[u] = alpha * __uint_as_float(r[u]);
                if (beta != 0.f && cin_ok) {
                    const uint8_t* cb = cbox + cl * kBoxBytes;
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 v = *reinterpret_cast<const float4*>(cb + lane * 128 + ((c4 ^ (lane & 7)) << 4));
                        out[4 * c4 + 0] += v.x;
                        out[4 * c4 + 1] += v.y;
                        out[4 * c4 + 2] += v.z;
                        out[4 * c4 + 3] += v.w;
                    }
                }
                // outputs: each 32x32 block through a swizzled box in shared memory and one TMA
                // store.  Boxes: this chunk's C box (read above), the staging box, and for the
                // second chunk also the first chunk's C box; a box is rewritten only after the
                // TMA has read it.
                __syncwarp();   // every lane has read its C row before the boxes are rewritten
                uint8_t* box[3] = {cbox + cl * kBoxBytes, kb, cbox};
                const int nbox = cl == 0 ? 2 : 3;
                const int j0 = (int)(c_col0 + 32 * c);
                int nb = 0;
                auto put = [&](const float (&v)[32], bool transposed, const CUtensorMap* map, int x, int y,
                               bool in_range) {
                    if (nb == nbox) {   // out of boxes: wait until the TMA has read them
                        if (lane == 0) {
                            bulk_commit();
                            bulk_wait_read<0>();
                        }
                        __syncwarp();
                        nb = 0;
                    }
                    uint8_t* bx = box[nb++];
                    if (transposed)
                        box_put_col(bx, lane, v);
                    else
                        box_put_row(bx, lane, v);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && in_range) tma_store_2d(map, bx, x, y);
                };
                if (C) put(out, false, mc_store, j0, i0, i0 < c_rows && j0 < c_cols);
                if (s_split || t_hi) {
                    float hi[32], lo[32];
#pragma unroll
                    for (int u = 0; u < 32; ++u) split_tf32(out[u], hi[u], lo[u]);
                    if (s_split) {
                        put(hi, false, &maps.rs_hi32, (int)(s_col0 + 32 * c), i0, true);
                        put(lo, false, &maps.rs_lo32, (int)(s_col0 + 32 * c), i0, true);
                    }
                    if (t_hi) {
                        put(hi, true, t_hi, i0, (int)(t_row0 + 32 * c), true);
                        put(lo, true, t_lo, i0, (int)(t_row0 + 32 * c), true);
                    }
                }
                if (lane == 0) {
                    bulk_commit();
                    if (cl == 0) bulk_wait_read<0>();   // the boxes are rewritten by the second chunk
                }
                __syncwarp();
            }
            if (lane == 0) {
                bulk_wait<0>();            // this warp's stores are complete
                fence_proxy_async_global();
            }
            __syncwarp();
            // completion: the stores of all four warps, then the counter
            if (warp == 2 && lane == 0) DAG_TRACE(16 * T + 8 * (long long)tk.t + 6, globaltimer_ns());
            named_bar_epi();
            if (warp == 2 && lane == 0) {   // release: the four warps' stores, then the counter
                fence_proxy_async_global();
                __threadfence();
                if (ok && cin_ok) atomicAdd(dag_done_ctr(g, tk), 1);
                else atomicExch(abort, 1);
                DAG_TRACE(16 * T + 8 * (long long)tk.t + 4, globaltimer_ns());
                mbar_arrive(&ctl.task_empty[s]);
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

inline long long chol_n(long long d) { return (d + gq::NB - 1) / gq::NB * gq::NB; }

struct HinvWs {
    float *A, *S, *RS_hi, *RS_lo, *UT_hi, *UT_lo, *TT_hi, *TT_lo, *Xd_hi, *Xd_lo, *scal;
    int* ctr;
    int* rank;   // inverse of a caller's permutation (permuted factorization only)
};

inline size_t hinv_ws_bytes(long long d) {
    const long long n = chol_n(d), T = n / gq::NB;
    return (size_t)(8 * n * n + 2 * n * gq::NB + 64) * sizeof(float) +
           (size_t)(gq::dag_ctr_ints((int)T) + n) * sizeof(int);
}

inline HinvWs hinv_ws_carve(void* ws, long long d) {
    const long long n = chol_n(d), T = n / gq::NB;
    float* p = static_cast<float*>(ws);
    HinvWs w;
    float** big[] = {&w.A, &w.S, &w.RS_hi, &w.RS_lo, &w.UT_hi, &w.UT_lo, &w.TT_hi, &w.TT_lo};
    for (float** b : big) {
        *b = p;
        p += n * n;
    }
    w.Xd_hi = p;
    p += n * gq::NB;
    w.Xd_lo = p;
    p += n * gq::NB;
    w.scal = p;
    p += 64;
    w.ctr = reinterpret_cast<int*>(p);
    w.rank = w.ctr + gq::dag_ctr_ints((int)T);
    return w;
}

// Enqueue the whole factorization on stream st: lambda, the damped copy (with the first
// panel's split), the public U's strictly lower blocks zeroed, the counters cleared, then
// the persistent kernel (one CTA per SM).
inline cudaError_t hinv_run(const float* H, long long d, float damp_rel, float* U, void* ws, cudaStream_t st,
                            const int* perm = nullptr) {
    const long long n = chol_n(d);
    const int T = (int)(n / gq::NB);
    HinvWs w = hinv_ws_carve(ws, d);
    {
        gqh::TimedScope ts__("diag_mean", st);
        gq::diag_mean_kernel<<<1, 1024, 0, st>>>(H, d, damp_rel, w.scal);
    }
    GQ_TRY(cudaGetLastError());
    if (perm) {   // factor P^T Hd P: validate the permutation, then a gathering damped copy
        GQ_TRY(cudaMemsetAsync(w.rank, 0xFF, (size_t)d * sizeof(int), st));
        {
            gqh::TimedScope ts__("perm_invert", st);
            gq::perm_invert_kernel<<<(unsigned)((d + 255) / 256), 256, 0, st>>>(perm, d, w.rank);
        }
        GQ_TRY(cudaGetLastError());
        {
            gqh::TimedScope ts__("damp_copy_perm", st);
            gq::damp_copy_perm_kernel<<<(unsigned)n, 256, 0, st>>>(H, perm, d, n, w.scal, w.A, w.RS_hi, w.RS_lo, U,
                                                                   w.ctr, (int)gq::dag_ctr_ints((int)T));
        }
        GQ_TRY(cudaGetLastError());
    } else {
        {
            gqh::TimedScope ts__("damp_copy", st);
            gq::damp_copy_kernel<<<(unsigned)(T * T), 256, 0, st>>>(H, d, n, w.scal, w.A, w.RS_hi, w.RS_lo, U, w.ctr,
                                                        (int)gq::dag_ctr_ints((int)T));
        }
        GQ_TRY(cudaGetLastError());
    }
    const uint64_t N = (uint64_t)n;
    gq::DagMaps m;
    if (!make_tmap_2d(&m.rs_hi, w.RS_hi, 4, N, N, N, gq::BM, 32) || !make_tmap_2d(&m.rs_lo, w.RS_lo, 4, N, N, N, gq::BM, 32) ||
        !make_tmap_2d(&m.xd_hi, w.Xd_hi, 4, N, gq::NB, gq::NB, gq::BM, 32) ||
        !make_tmap_2d(&m.xd_lo, w.Xd_lo, 4, N, gq::NB, gq::NB, gq::BM, 32) ||
        !make_tmap_2d(&m.tt_hi, w.TT_hi, 4, N, N, N, gq::BM, 32) || !make_tmap_2d(&m.tt_lo, w.TT_lo, 4, N, N, N, gq::BM, 32) ||
        !make_tmap_2d(&m.ut_hi, w.UT_hi, 4, N, N, N, gq::BM, 32) || !make_tmap_2d(&m.ut_lo, w.UT_lo, 4, N, N, N, gq::BM, 32) ||
        !make_tmap_2d(&m.ca, w.A, 4, N, N, N, 32, 32) || !make_tmap_2d(&m.cs, w.S, 4, N, N, N, 32, 32) ||
        !make_tmap_2d(&m.rs_hi32, w.RS_hi, 4, N, N, N, 32, 32) || !make_tmap_2d(&m.rs_lo32, w.RS_lo, 4, N, N, N, 32, 32) ||
        !make_tmap_2d(&m.ut_hi32, w.UT_hi, 4, N, N, N, 32, 32) || !make_tmap_2d(&m.ut_lo32, w.UT_lo, 4, N, N, N, 32, 32) ||
        !make_tmap_2d(&m.tt_hi32, w.TT_hi, 4, N, N, N, 32, 32) || !make_tmap_2d(&m.tt_lo32, w.TT_lo, 4, N, N, N, 32, 32) ||
        !make_tmap_2d(&m.u32, U, 4, (uint64_t)d, (uint64_t)d, (uint64_t)d, 32, 32))
        return cudaErrorInvalidValue;
    gq::DagArgs a{};
    a.T = T;
    a.n = n;
    a.d = d;
    a.A = w.A;
    a.S = w.S;
    a.RS_hi = w.RS_hi;
    a.RS_lo = w.RS_lo;
    a.Xd_hi = w.Xd_hi;
    a.Xd_lo = w.Xd_lo;
    a.UT_hi = w.UT_hi;
    a.UT_lo = w.UT_lo;
    a.TT_hi = w.TT_hi;
    a.TT_lo = w.TT_lo;
    a.U = U;
    a.ctr = w.ctr;
    GQ_TRY(ensure_smem_attr(reinterpret_cast<const void*>(gq::chol_dag_kernel), gq::DAG_SMEM));
    // one CTA per SM (the shared memory allows no second); a single tile needs only the leaf
    const unsigned grid = T == 1 ? 1u : (unsigned)std::min<long long>(num_sms(), 1 + gq::dag_total_tasks(T));
    {
        gqh::TimedScope ts__("chol_dag", st);
        GQ_TRY(launch_plain(gq::chol_dag_kernel, dim3(grid), dim3(gq::DAG_BLOCK), (size_t)gq::DAG_SMEM, st, m,
                            (const gq::DagArgs)a));
    }
    return cudaGetLastError();
}

}  // namespace gqh
