// plan.cu -- split-KV work planner for the decode calls.
//
// Every (shard n, request b) owns count_n(L_b) local tokens.  The planner cuts
// each into chunks of at most C tokens (C a multiple of the kernel's token
// granule, at least total_tokens / target_units), so the persistent decode
// grid sees many similar-sized units regardless of the length mix, and lists
// the units longest-first (bucketed by floor(log2(length))).
//
// Units are gathered into output groups; a group with several units gives each
// a split-partial slot and its last unit to finish LSE-merges them (the
// arithmetic of "Efficient Decode Context Parallelism with vLLM for Long
// Context Workloads", section 4.1, which the all-gather + reduce-scatter of
// the pages performs across GPUs):
//  - per-shard partials: one group per (n, b), output row block n*B + b;
//  - merged output: one group per request b, output row block b, merged in two
//    levels: the last chunk of a shard cut into several chunks merges that
//    shard's chunks, and the last shard of the request to complete merges the
//    shards' partials.  No merge reads more than max(chunks per shard, N)
//    partials, so a long request does not leave one CTA a merge of hundreds.
//    The request's units are listed next to each other, so they run at the
//    same time on different SMs and the merges find the partials still in L2.
//    Empty shards add no unit; a request with no token at all gets one empty
//    unit (O = 0, LSE = -inf).
#include "common.cuh"
#include "kernels.h"

namespace dcp {

namespace {

constexpr int kPlanThreads = 1024;

__device__ __forceinline__ int length_bucket(int64_t len) {
    return len <= 0 ? 32 : __clzll((unsigned long long)len) - 32;
}

// inclusive block scan of one int per thread; returns the inclusive value and the block total
__device__ int block_scan_incl(int v, int* total, int* warp_sums) {
    int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) warp_sums[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += t;
        }
        warp_sums[lane] = w;
    }
    __syncthreads();
    int r = v + (warp > 0 ? warp_sums[warp - 1] : 0);
    *total = warp_sums[31];
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ seq_lens, int B, int N, int I,
                                                            int q_len, int merged, int shard_lo, int shard_hi,
                                                            int granule, int min_chunk, int target_units, int n_hb,
                                                            uint8_t* ws, WsLayout lay, int64_t* finish_ns,
                                                            int* status) {
    PlanHeader* hdr = reinterpret_cast<PlanHeader*>(ws);
    Unit* units = reinterpret_cast<Unit*>(ws + lay.off_units);
    int32_t* done = reinterpret_cast<int32_t*>(ws + lay.off_done);
    int32_t* grp_k = reinterpret_cast<int32_t*>(ws + lay.off_k);       // units per group [groups]
    int32_t* slot_base = reinterpret_cast<int32_t*>(ws + lay.off_base);  // first split slot per group

    __shared__ unsigned long long s_total;
    __shared__ int s_hist[33];
    __shared__ int s_cursor[33];
    __shared__ int s_warp[32];
    __shared__ int s_units_total;
    __shared__ int s_split_total;
    const int tid = threadIdx.x;
    if (tid == 0) {
        hdr->t_start_ns = (int64_t)global_timer_ns();
        s_total = 0;
        s_units_total = 0;
        s_split_total = 0;
    }
    if (tid < 33) s_hist[tid] = 0;
    __syncthreads();

    // 1. total tokens
    unsigned long long t = 0;
    for (int b = tid; b < B; b += kPlanThreads) {
        int L = seq_lens[b];
        if (L < 0 || (L > 0 && L < q_len)) record_status(status, DCP_ERR_INVALID_ARG);
        t += (unsigned long long)(L < 0 ? 0 : L);
    }
    atomicAdd(&s_total, t);
    __syncthreads();
    const int64_t T = (int64_t)s_total;

    // 2. chunk size
    int64_t C = (T + target_units - 1) / (target_units > 0 ? target_units : 1);
    if (C < min_chunk) C = min_chunk;
    C = (C + granule - 1) / granule * granule;
    if (C > (1 << 30)) C = 1 << 30;

    // 3. units per group, split-slot scan, length histogram (a request's units share
    //    one bucket in merged mode: that of its longest unit)
    const int NG = merged ? B : N * B;
    for (int i = tid; i < (N + 1) * B * n_hb; i += kPlanThreads) done[i] = 0;
    if (finish_ns)
        for (int i = tid; i < NG; i += kPlanThreads) finish_ns[i] = 0;
    int units_local = 0;
    int carry = 0;
    for (int base = 0; base < NG; base += kPlanThreads) {
        const int gi = base + tid;
        int k = 0, split = 0;
        if (gi < NG) {
            if (merged) {
                // slots: one per shard with tokens when there are two or more, plus one per
                // chunk of every shard cut into several chunks
                const int L = max(seq_lens[gi], 0);
                int64_t cmax = 0;
                int m = 0;
                for (int n = shard_lo; n < shard_hi; n++) {
                    const int64_t cnt = count_of(L, N, I, n);
                    const int kn = (int)((cnt + C - 1) / C);
                    k += kn;
                    split += kn >= 2 ? kn : 0;
                    m += cnt > 0 ? 1 : 0;
                    cmax = cnt > cmax ? cnt : cmax;
                }
                split += m >= 2 ? m : 0;
                if (k == 0) k = 1;
                atomicAdd(&s_hist[cmax > 0 ? length_bucket(cmax < C ? cmax : C) : 32], k);
            } else {
                const int n = gi / B, b = gi - n * B;
                const int L = seq_lens[b];
                const int64_t cnt = count_of(L < 0 ? 0 : L, N, I, n);
                k = cnt == 0 ? 1 : (int)((cnt + C - 1) / C);
                if (cnt > 0) {
                    if (k > 1) atomicAdd(&s_hist[length_bucket(C)], k - 1);
                    atomicAdd(&s_hist[length_bucket(cnt - (int64_t)(k - 1) * C)], 1);
                } else {
                    atomicAdd(&s_hist[32], 1);
                }
            }
            grp_k[gi] = k;
            if (!merged) split = k >= 2 ? k : 0;
            units_local += k;
        }
        int total;
        int incl = block_scan_incl(split, &total, s_warp);
        if (gi < NG) slot_base[gi] = carry + incl - split;
        carry += total;
    }
    atomicAdd(&s_units_total, units_local);
    __syncthreads();
    if (tid == 0) {
        s_split_total = carry;
        int acc = 0;
        for (int i = 0; i < 33; i++) {
            s_cursor[i] = acc;
            acc += s_hist[i];
        }
    }
    __syncthreads();
    const int n_units = s_units_total;
    const bool fits = n_units <= lay.max_units && s_split_total <= lay.max_split;
    if (tid == 0) {
        hdr->num_units = fits ? n_units : 0;
        hdr->chunk_tokens = (int32_t)C;
        hdr->max_units = lay.max_units;
        hdr->max_split = lay.max_split;
        hdr->total_tokens = T;
        hdr->next_unit = 0;
        hdr->merged = merged;
        if (!fits) record_status(status, DCP_ERR_WORKSPACE_TOO_SMALL);
    }
    if (!fits) return;

    // 4. emit units, longest bucket first
    if (merged) {
        for (int b = tid; b < B; b += kPlanThreads) {
            const int L = max(seq_lens[b], 0);
            const int k = grp_k[b];
            int64_t cmax = 0;
            int m = 0;
            for (int n = shard_lo; n < shard_hi; n++) {
                const int64_t cnt = count_of(L, N, I, n);
                cmax = cnt > cmax ? cnt : cmax;
                m += cnt > 0 ? 1 : 0;
            }
            const int pos = atomicAdd(&s_cursor[cmax > 0 ? length_bucket(cmax < C ? cmax : C) : 32], k);
            Unit u;
            u.b = b;
            u.grp = b;
            u.n_sh = m >= 2 ? m : 1;
            u.sslot_base = m >= 2 ? slot_base[b] : -1;
            u.pad = 0;
            if (cmax == 0) {  // a request with no token: one empty unit
                u.n = shard_lo;
                u.t0 = u.t1 = 0;
                u.slot = -1;
                u.n_chunks = 1;
                u.slot_base = -1;
                u.sslot = -1;
                units[pos] = u;
                continue;
            }
            int next_slot = slot_base[b] + (m >= 2 ? m : 0);  // chunk slots follow the shard slots
            int j = 0, i = 0;
            for (int n = shard_lo; n < shard_hi; n++) {
                const int64_t cnt = count_of(L, N, I, n);
                if (cnt == 0) continue;
                const int kn = (int)((cnt + C - 1) / C);
                u.n = n;
                u.n_chunks = kn;
                u.slot_base = kn >= 2 ? next_slot : -1;
                u.sslot = m >= 2 ? slot_base[b] + i : -1;
                for (int c = 0; c < kn; c++, j++) {
                    const int64_t t0 = (int64_t)c * C;
                    u.t0 = (int32_t)t0;
                    u.t1 = (int32_t)(t0 + C < cnt ? t0 + C : cnt);
                    u.slot = kn >= 2 ? next_slot + c : -1;
                    units[pos + j] = u;
                }
                if (kn >= 2) next_slot += kn;
                i++;
            }
        }
        return;
    }
    for (int s = tid; s < NG; s += kPlanThreads) {
        int n = s / B, b = s - n * B;
        int L = seq_lens[b];
        int64_t cnt = count_of(L < 0 ? 0 : L, N, I, n);
        int k = grp_k[s];
        int sb = slot_base[s];
        for (int j = 0; j < k; j++) {
            int64_t t0 = (int64_t)j * C;
            int64_t t1 = t0 + C < cnt ? t0 + C : cnt;
            int pos = atomicAdd(&s_cursor[length_bucket(t1 - t0)], 1);
            Unit u;
            u.n = n;
            u.b = b;
            u.t0 = (int32_t)t0;
            u.t1 = (int32_t)t1;
            u.slot = k >= 2 ? sb + j : -1;
            u.n_chunks = k;
            u.slot_base = k >= 2 ? sb : -1;
            u.grp = s;
            u.sslot = -1;
            u.n_sh = 1;
            u.sslot_base = -1;
            u.pad = 0;
            units[pos] = u;
        }
    }
}

}  // namespace

cudaError_t launch_plan(const int32_t* seq_lens, int B, int N, int I, int q_len, int merged, int shard_lo,
                        int shard_hi, int granule, int min_chunk, int target_units, int n_hb, void* ws, int max_units,
                        int max_split, int hq, int dv, int64_t* finish_ns, int* status, cudaStream_t s) {
    WsLayout lay = ws_layout(N, B, hq, dv, max_units, max_split);
    plan_kernel<<<1, kPlanThreads, 0, s>>>(seq_lens, B, N, I, q_len, merged, shard_lo, shard_hi, granule, min_chunk,
                                           target_units, n_hb, reinterpret_cast<uint8_t*>(ws), lay, finish_ns, status);
    return cudaGetLastError();
}

}  // namespace dcp
