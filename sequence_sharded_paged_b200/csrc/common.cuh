// common.cuh -- device helpers shared by the libdcp kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dcp.h"

namespace dcp {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// A kernel that waits longer than this on one copy gives up (DCP_ERR_TIMEOUT).
constexpr uint64_t kWaitLimitNs = 4000000000ull;

// ---------------------------------------------------------------------------
// sticky device status word
// ---------------------------------------------------------------------------
__device__ __forceinline__ void record_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------------------
// shard map arithmetic (owner = (p / I) mod N; owned positions packed in order)
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int owner_of(int64_t p, int N, int I) { return (int)((p / I) % N); }

__host__ __device__ __forceinline__ int64_t local_of(int64_t p, int N, int I) {
    return (p / ((int64_t)I * N)) * I + p % I;
}

__host__ __device__ __forceinline__ int64_t count_of(int64_t L, int N, int I, int n) {
    int64_t IN = (int64_t)I * N;
    int64_t r = L % IN - (int64_t)n * I;
    r = r < 0 ? 0 : (r > I ? I : r);
    return (L / IN) * I + r;
}

// ---------------------------------------------------------------------------
// shared memory / mbarrier / bulk copy
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking: has the phase with parity `parity` of `bar` completed?
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete.  Gives up after kWaitLimitNs
// (records DCP_ERR_TIMEOUT, sets *abort) and returns false.  Returns false
// immediately when *abort is already set by another warp.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (abort && *abort) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            record_status(status, DCP_ERR_TIMEOUT);
            if (abort) *abort = 1;
            return false;
        }
    }
}

// 1-D bulk copy global -> shared, completion counted on `bar` (bytes % 16 == 0,
// both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// L2 eviction-priority hint variant: the KV stream is read exactly once.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void bulk_g2s_hint(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
        "%4;" ::"r"(smem_u32(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// ---------------------------------------------------------------------------
// conversions
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// two e4m3 bytes (low half of `w`) -> two floats, exact
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t w) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)w, __NV_E4M3);
    return __half22float2(*reinterpret_cast<__half2*>(&h));
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------------------
// work units produced by the planner
// ---------------------------------------------------------------------------
struct Unit {
    int32_t n;          // shard
    int32_t b;          // request
    int32_t t0, t1;     // local token range [t0, t1) of shard n of request b
    int32_t slot;       // split-partial slot of this chunk, -1 when the shard is one chunk
    int32_t n_chunks;   // chunks of this shard
    int32_t slot_base;  // first split slot of this shard
    int32_t grp;        // output row block of this shard: (n - first decoded shard) * B + b
};
static_assert(sizeof(Unit) == 32, "Unit layout");

struct PlanHeader {
    int32_t num_units;
    int32_t chunk_tokens;
    int32_t max_units;
    int32_t max_split;
    int64_t total_tokens;
    int32_t next_unit;  // dynamic-scheduling ticket (zeroed by the planner)
    int32_t pad;
    int64_t t_start_ns; // %globaltimer when the planner started
};

// Per-stage metadata of the dynamically scheduled kernels: which unit and
// token a ring stage holds.  Written by the producer before it arrives on the
// stage's full barrier.
struct StageMeta {
    int32_t unit;   // unit index, -1 = no more work
    int32_t t;      // first local token of the stage
    int32_t flags;  // kStageFirst | kStageLast | kStageValid
    int32_t sidx;   // stage index within the unit
};
__device__ __forceinline__ StageMeta load_meta(const StageMeta* m) {
    const volatile int32_t* v = reinterpret_cast<const volatile int32_t*>(m);
    return StageMeta{v[0], v[1], v[2], v[3]};
}
constexpr int kStageFirst = 1;
constexpr int kStageLast = 2;
constexpr int kStageValid = 4;

// Workspace layout (all offsets 256-byte aligned):
//   PlanHeader | Unit[max_units] | int32 done[N*B*hq] | int32 shard_k[N*B] |
//   int32 slot_base[N*B] | float split_o[max_split][hq][dv] | float split_lse[max_split][hq]
// done: chunk counters per (shard, request, head block).
struct WsLayout {
    size_t off_units, off_done, off_k, off_base, off_split_o, off_split_lse, total;
    int32_t max_units, max_split;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

__host__ inline WsLayout ws_layout(int N, int B, int hq, int dv, int max_units, int max_split) {
    WsLayout w;
    size_t o = align256(sizeof(PlanHeader));
    w.off_units = o;
    o = align256(o + sizeof(Unit) * (size_t)max_units);
    w.off_done = o;  // one counter per (shard, request, head block); head blocks <= hq
    o = align256(o + sizeof(int32_t) * (size_t)N * B * hq);
    w.off_k = o;
    o = align256(o + sizeof(int32_t) * (size_t)N * B);
    w.off_base = o;
    o = align256(o + sizeof(int32_t) * (size_t)N * B);
    w.off_split_o = o;
    o = align256(o + sizeof(float) * (size_t)max_split * hq * dv);
    w.off_split_lse = o;
    o = align256(o + sizeof(float) * (size_t)max_split * hq);
    w.total = o;
    w.max_units = max_units;
    w.max_split = max_split;
    return w;
}

// Everything a decode kernel needs to locate its units and outputs.
struct DecodeArgs {
    // cache
    const uint8_t* k_pages;
    const uint8_t* v_pages;
    const float* kv_scales;
    const int32_t* block_tables;
    int32_t n_shards, interleave, page_size, num_pages, batch, max_local_pages;
    int32_t hq, hkv, dk, dv;
    float scale_log2;  // softmax scale * log2(e)
    // inputs / outputs
    const __nv_bfloat16* q;
    const int32_t* seq_lens;
    float* o_partial;
    float* lse;
    // workspace
    const PlanHeader* plan;
    int32_t* ticket;  // &plan->next_unit
    const Unit* units;
    int32_t* done;
    float* split_o;
    float* split_lse;
    uint8_t* qs;         // fp8 MLA: query rows split into two e4m3 terms [B][128][576] (else null)
    float* qinv;         // fp8 MLA: 1 / sigma per (request, head) [B][64] (else null)
    int* status;
    // several query tokens per request: hq counts query ROWS (q_len x heads), row
    // r = j * (hq / q_len) + head belongs to query token j
    int32_t q_len;
    int64_t* finish_ns;  // per request: ns from the planner's start until its last shard is decoded (or null)
    // first shard whose block tables are present: 0 when block_tables holds every
    // shard ([N][B][max_local_pages]); r when it holds only shard r's ([1][B][..]),
    // the cache of rank r of a multi-GPU group
    int32_t bt_shard0;
};

// Local tokens [0, limit) of shard u.n that query token j attends: the positions
// p <= L_b - q_len + j (causal among the q_len new tokens, which are the last
// positions of the request).  With one query token every owned token is attended.
__device__ __forceinline__ int row_limit(const DecodeArgs& a, const Unit& u, int j) {
    if (a.q_len <= 1) return 0x7fffffff;
    const int L = __ldg(a.seq_lens + u.b) - a.q_len + j + 1;
    return L <= 0 ? 0 : (int)count_of(L, a.n_shards, a.interleave, u.n);
}

// Completion time of request b (call after a shard's result of b is stored; the
// planner zeroes the array and the last shard to finish sets it).
__device__ __forceinline__ void record_finish(const DecodeArgs& a, int b) {
    if (!a.finish_ns) return;
    const uint64_t dt = global_timer_ns() - (uint64_t)a.plan->t_start_ns;
    atomicMax(reinterpret_cast<unsigned long long*>(a.finish_ns + b), (unsigned long long)dt);
}

// Invalidate the 128-byte L2 line at p (128-byte aligned) without writing it
// back: for scratch data that has been read for the last time.
__device__ __forceinline__ void discard_l2_line(const void* p) {
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

// Fetch the physical page of local page j of (n, b); -1 when invalid.
__device__ __forceinline__ int page_of(const DecodeArgs& a, int n, int b, int j) {
    if (j >= a.max_local_pages) return -1;
    int pg = __ldg(a.block_tables + ((int64_t)(n - a.bt_shard0) * a.batch + b) * a.max_local_pages + j);
    return (pg >= 0 && pg < a.num_pages) ? pg : -1;
}

}  // namespace dcp
