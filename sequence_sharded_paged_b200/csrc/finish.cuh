// finish.cuh -- end of one work unit: store a shard's partial, or a chunk's
// split partial and, in the last chunk of the shard to finish, the LSE merge
// of the chunks (split-KV reduce).  The merge is the arithmetic of
// "Efficient Decode Context Parallelism with vLLM for Long Context Workloads",
// section 4.1 (LSE-reweighted sum of partials), applied within one shard.
#pragma once

#include "common.cuh"

namespace dcp {

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Merge the K partials in split slots [base, base + K) for rows h0..h0+nh-1
// into dst_o [rows][dv] / dst_lse [rows] (rows indexed from 0), executed by
// warps w0, w0 + 1, .., w0 + nw - 1 of the caller (one warp per row, lane =
// tid & 31):
//   M = max_j lse_j,  O = sum_j exp(lse_j - M) O_j / sum_j exp(lse_j - M),
//   LSE = M + ln sum_j exp(lse_j - M).
// The partials are dead afterwards, so each warp discards the L2 lines it has
// read: a merge that runs while they are still in L2 keeps them from ever
// reaching HBM.
__device__ inline void merge_slots(const DecodeArgs& a, int base, int K, int h0, int nh, float* dst_o,
                                   float* dst_lse, int w, int nw, int lane) {
    constexpr int kMaxV = 4;  // float4 per lane and row: dv <= 512
    const int dv = a.dv;
    const int nv = dv / 4;
    for (int h = w; h < nh; h += nw) {
        const float* lse_col = a.split_lse + (int64_t)base * a.hq + h0 + h;
        float M = -INFINITY;
        for (int j = lane; j < K; j += 32) M = fmaxf(M, __ldcg(lse_col + (int64_t)j * a.hq));
#pragma unroll
        for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float wsum = 0.f;
        if (M != -INFINITY)
            for (int j = lane; j < K; j += 32) {
                const float lj = __ldcg(lse_col + (int64_t)j * a.hq);
                wsum += lj == -INFINITY ? 0.f : expf(lj - M);
            }
#pragma unroll
        for (int o = 16; o; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
        float4 acc[kMaxV];
#pragma unroll
        for (int r = 0; r < kMaxV; r++) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (M != -INFINITY) {
#pragma unroll 8
            for (int j = 0; j < K; j++) {
                const float lj = __ldcg(lse_col + (int64_t)j * a.hq);
                const float4* src =
                    reinterpret_cast<const float4*>(a.split_o + ((int64_t)(base + j) * a.hq + h0 + h) * dv);
                float4 x[kMaxV];
#pragma unroll
                for (int r = 0; r < kMaxV; r++)
                    x[r] = (lane + 32 * r < nv) ? __ldcg(src + lane + 32 * r) : make_float4(0.f, 0.f, 0.f, 0.f);
                const float wj = lj == -INFINITY ? 0.f : expf(lj - M);
#pragma unroll
                for (int r = 0; r < kMaxV; r++) {
                    acc[r].x = fmaf(wj, x[r].x, acc[r].x);
                    acc[r].y = fmaf(wj, x[r].y, acc[r].y);
                    acc[r].z = fmaf(wj, x[r].z, acc[r].z);
                    acc[r].w = fmaf(wj, x[r].w, acc[r].w);
                }
            }
        }
        const float inv = M != -INFINITY ? 1.f / wsum : 0.f;
        float4* dst = reinterpret_cast<float4*>(dst_o + (int64_t)(h0 + h) * dv);
#pragma unroll
        for (int r = 0; r < kMaxV; r++)
            if (lane + 32 * r < nv)
                __stcg(dst + lane + 32 * r, make_float4(acc[r].x * inv, acc[r].y * inv, acc[r].z * inv, acc[r].w * inv));
        if (lane == 0) __stcg(dst_lse + h0 + h, (M == -INFINITY) ? -INFINITY : M + logf(wsum));
        // every lane has consumed its loads of this row (the values are stored above)
        __syncwarp();
        const int lines = dv / 32;  // 128-byte lines per row of dv floats
        for (int i = lane; i < K * lines; i += 32) {
            const int j = i / lines, l = i - j * lines;
            discard_l2_line(a.split_o + ((int64_t)(base + j) * a.hq + h0 + h) * dv + l * 32);
        }
    }
}

// The output row block of the unit's shard.
__device__ __forceinline__ float* shard_out(const DecodeArgs& a, const Unit& u) {
    return a.o_partial + (int64_t)u.grp * a.hq * a.dv;
}
__device__ __forceinline__ float* shard_lse(const DecodeArgs& a, const Unit& u) {
    return a.lse + (int64_t)u.grp * a.hq;
}

// Executed by the NT threads of barrier `bar_id` (tid in [0, NT), NT a
// multiple of 32).
//  sO   [nh][dv] normalised output of this unit for rows h0..h0+nh-1 (smem)
//  sLse [nh]     natural-log LSE (-inf when the unit saw no token)
//  hb / n_hb     head block of this unit and head blocks per unit (split counters
//                are per (shard, head block))
// Records the request's completion time (a.finish_ns) when this completes the shard.
template <int NT>
__device__ void finish_unit(const DecodeArgs& a, const Unit& u, int hb, int n_hb, int h0, int nh,
                            const float* sO, const float* sLse, int* s_flag, int tid, int bar_id) {
    const int dv = a.dv;
    const int nvec = nh * dv / 4;
    if (u.n_chunks == 1) {
        float4* dst = reinterpret_cast<float4*>(shard_out(a, u) + (int64_t)h0 * dv);
        const float4* src = reinterpret_cast<const float4*>(sO);
        for (int i = tid; i < nvec; i += NT) dst[i] = src[i];
        for (int i = tid; i < nh; i += NT) shard_lse(a, u)[h0 + i] = sLse[i];
        if (a.finish_ns) {
            named_barrier_sync(bar_id, NT);
            if (tid == 0) record_finish(a, u.b);
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
        int old = atomicAdd(a.done + (int64_t)u.grp * n_hb + hb, 1);
        *s_flag = (old == u.n_chunks - 1) ? 1 : 0;
    }
    named_barrier_sync(bar_id, NT);
    const int last = *(volatile int*)s_flag;
    named_barrier_sync(bar_id, NT);
    if (!last) return;
    __threadfence();
    merge_slots(a, u.slot_base, u.n_chunks, h0, nh, shard_out(a, u), shard_lse(a, u), tid >> 5, NT >> 5, tid & 31);
    if (a.finish_ns) {
        named_barrier_sync(bar_id, NT);
        if (tid == 0) record_finish(a, u.b);
    }
}

}  // namespace dcp
