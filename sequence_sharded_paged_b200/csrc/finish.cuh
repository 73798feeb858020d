// finish.cuh -- end of one work unit: store the unit's output when its group
// has one unit, or its split partial and, in the last unit of the group to
// finish, the LSE merge of the group's units.  A group is the chunks of one
// shard (per-shard partials, the split-KV reduce) or the chunks of every
// shard of one request (merged output).  The merge is the arithmetic of
// "Efficient Decode Context Parallelism with vLLM for Long Context Workloads",
// section 4.1 (LSE-reweighted sum of partials).
#pragma once

#include "common.cuh"

namespace dcp {

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Merge the split partials of the units of group u.grp for rows h0..h0+nh-1
// into o_partial / lse (executed by the NT threads of barrier `bar_id`, tid in
// [0, NT)):
//   M = max_j lse_j,  O = sum_j exp(lse_j - M) O_j / sum_j exp(lse_j - M),
//   LSE = M + ln sum_j exp(lse_j - M).
// The partials are dead afterwards, so their L2 lines are discarded: a merge
// that runs while they are still in L2 keeps them from ever reaching HBM.
__device__ inline void merge_split_chunks(const DecodeArgs& a, const Unit& u, int h0, int nh, int tid, int NT,
                                          int bar_id) {
    const int dv = a.dv;
    const int K = u.n_chunks;
    const int64_t grp = u.grp;
    for (int i = tid; i < nh * (dv / 4); i += NT) {
        const int h = i / (dv / 4), d4 = i - h * (dv / 4);
        const float* lse_col = a.split_lse + (int64_t)u.slot_base * a.hq + h0 + h;
        float M = -INFINITY;
        for (int j = 0; j < K; j++) M = fmaxf(M, __ldcg(lse_col + (int64_t)j * a.hq));
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        float wsum = 0.f;
        if (M != -INFINITY) {
            for (int j = 0; j < K; j++) {
                const float lj = __ldcg(lse_col + (int64_t)j * a.hq);
                if (lj == -INFINITY) continue;
                const float w = expf(lj - M);
                wsum += w;
                const float4 x = __ldcg(
                    reinterpret_cast<const float4*>(a.split_o + ((int64_t)(u.slot_base + j) * a.hq + h0 + h) * dv) + d4);
                o.x += w * x.x;
                o.y += w * x.y;
                o.z += w * x.z;
                o.w += w * x.w;
            }
            const float inv = 1.f / wsum;
            o.x *= inv;
            o.y *= inv;
            o.z *= inv;
            o.w *= inv;
        }
        reinterpret_cast<float4*>(a.o_partial + (grp * a.hq + h0 + h) * dv)[d4] = o;
        if (d4 == 0) a.lse[grp * a.hq + h0 + h] = (M == -INFINITY) ? -INFINITY : M + logf(wsum);
    }
    // every thread has consumed its loads (their values are stored above)
    named_barrier_sync(bar_id, NT);
    const int lines = dv / 32;  // 128-byte lines per row of dv floats
    const int n_lines = K * nh * lines;
    for (int i = tid; i < n_lines; i += NT) {
        const int j = i / (nh * lines), rem = i - j * nh * lines;
        const int h = rem / lines, l = rem - h * lines;
        discard_l2_line(a.split_o + ((int64_t)(u.slot_base + j) * a.hq + h0 + h) * dv + l * 32);
    }
}

// Executed by the NT threads of barrier `bar_id` (tid in [0, NT)).
//  sO   [nh][dv] normalised output of this unit for rows h0..h0+nh-1 (smem)
//  sLse [nh]     natural-log LSE (-inf when the unit saw no token)
//  hb / n_hb     head block of this unit and head blocks per unit (split counters
//                are per (group, head block))
// Records the group's completion time when a.finish_ns is set.
template <int NT>
__device__ void finish_unit(const DecodeArgs& a, const Unit& u, int hb, int n_hb, int h0, int nh,
                            const float* sO, const float* sLse, int* s_flag, int tid, int bar_id) {
    const int dv = a.dv;
    const int64_t grp = u.grp;
    const int nvec = nh * dv / 4;
    if (u.n_chunks == 1) {
        float4* dst = reinterpret_cast<float4*>(a.o_partial + (grp * a.hq + h0) * dv);
        const float4* src = reinterpret_cast<const float4*>(sO);
        for (int i = tid; i < nvec; i += NT) dst[i] = src[i];
        for (int i = tid; i < nh; i += NT) a.lse[grp * a.hq + h0 + i] = sLse[i];
        if (a.finish_ns) {
            named_barrier_sync(bar_id, NT);
            if (tid == 0) record_finish(a, (int)grp);
        }
        return;
    }
    {
        float4* dst = reinterpret_cast<float4*>(a.split_o + ((int64_t)u.slot * a.hq + h0) * dv);
        const float4* src = reinterpret_cast<const float4*>(sO);
        for (int i = tid; i < nvec; i += NT) __stcg(dst + i, src[i]);
        for (int i = tid; i < nh; i += NT) __stcg(a.split_lse + (int64_t)u.slot * a.hq + h0 + i, sLse[i]);
    }
    __threadfence();
    named_barrier_sync(bar_id, NT);
    if (tid == 0) {
        int old = atomicAdd(a.done + grp * n_hb + hb, 1);
        *s_flag = (old == u.n_chunks - 1) ? 1 : 0;
    }
    named_barrier_sync(bar_id, NT);
    const int last = *(volatile int*)s_flag;
    named_barrier_sync(bar_id, NT);
    if (!last) return;
    __threadfence();
    merge_split_chunks(a, u, h0, nh, tid, NT, bar_id);
    if (a.finish_ns) {
        named_barrier_sync(bar_id, NT);
        if (tid == 0) record_finish(a, (int)grp);
    }
}

}  // namespace dcp
