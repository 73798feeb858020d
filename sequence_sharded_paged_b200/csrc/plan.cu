// plan.cu -- split-KV work planner for the decode calls.
//
// Every (shard n, request b) owns count_n(L_b) local tokens.  The planner cuts
// each into chunks of at most C tokens (C a multiple of the kernel's token
// granule, at least total_tokens / target_units), so the persistent decode
// grid sees many similar-sized units regardless of the length mix, and lists
// the units longest-first (bucketed by floor(log2(length))).  Shards cut into
// several chunks get consecutive split-partial slots; the last chunk of such a
// shard to finish merges them (the LSE arithmetic of "Efficient Decode Context
// Parallelism with vLLM for Long Context Workloads", section 4.1, applied to
// the chunks of one shard).  Only shards [shard_lo, shard_hi) are planned: all
// of them on one GPU, or the one shard of a rank of a multi-GPU group.
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
                                                            int q_len, int shard_lo, int shard_hi, int granule,
                                                            int min_chunk, int target_units, int n_hb, uint8_t* ws,
                                                            WsLayout lay, int64_t* finish_ns, int* status) {
    PlanHeader* hdr = reinterpret_cast<PlanHeader*>(ws);
    Unit* units = reinterpret_cast<Unit*>(ws + lay.off_units);
    int32_t* done = reinterpret_cast<int32_t*>(ws + lay.off_done);
    int32_t* shard_k = reinterpret_cast<int32_t*>(ws + lay.off_k);
    int32_t* slot_base = reinterpret_cast<int32_t*>(ws + lay.off_base);

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

    // 1. total tokens of the planned shards
    const int NS = shard_hi - shard_lo;
    unsigned long long t = 0;
    for (int b = tid; b < B; b += kPlanThreads) {
        int L = seq_lens[b];
        if (L < 0 || (L > 0 && L < q_len)) record_status(status, DCP_ERR_INVALID_ARG);
        for (int n = shard_lo; n < shard_hi; n++) t += (unsigned long long)count_of(L < 0 ? 0 : L, N, I, n);
    }
    atomicAdd(&s_total, t);
    __syncthreads();
    const int64_t T = (int64_t)s_total;

    // 2. chunk size
    int64_t C = (T + target_units - 1) / (target_units > 0 ? target_units : 1);
    if (C < min_chunk) C = min_chunk;
    C = (C + granule - 1) / granule * granule;
    if (C > (1 << 30)) C = 1 << 30;

    // 3. chunks per shard, split-slot scan, length histogram
    const int NB = NS * B;
    for (int i = tid; i < NB * n_hb; i += kPlanThreads) done[i] = 0;
    if (finish_ns)
        for (int i = tid; i < B; i += kPlanThreads) finish_ns[i] = 0;
    int units_local = 0;
    int carry = 0;
    for (int base = 0; base < NB; base += kPlanThreads) {
        int s = base + tid;
        int k = 0, split = 0;
        if (s < NB) {
            int n = shard_lo + s / B, b = s % B;
            int L = seq_lens[b];
            int64_t cnt = count_of(L < 0 ? 0 : L, N, I, n);
            k = cnt == 0 ? 1 : (int)((cnt + C - 1) / C);
            shard_k[s] = k;
            split = k >= 2 ? k : 0;
            units_local += k;
            if (cnt > 0) {
                if (k > 1) atomicAdd(&s_hist[length_bucket(C)], k - 1);
                atomicAdd(&s_hist[length_bucket(cnt - (int64_t)(k - 1) * C)], 1);
            } else {
                atomicAdd(&s_hist[32], 1);
            }
        }
        int total;
        int incl = block_scan_incl(split, &total, s_warp);
        if (s < NB) slot_base[s] = carry + incl - split;
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
        if (!fits) record_status(status, DCP_ERR_WORKSPACE_TOO_SMALL);
    }
    if (!fits) return;

    // 4. emit units, longest bucket first
    for (int s = tid; s < NB; s += kPlanThreads) {
        int n = shard_lo + s / B, b = s % B;
        int L = seq_lens[b];
        int64_t cnt = count_of(L < 0 ? 0 : L, N, I, n);
        int k = shard_k[s];
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
            units[pos] = u;
        }
    }
}

}  // namespace

cudaError_t launch_plan(const int32_t* seq_lens, int B, int N, int I, int q_len, int shard_lo, int shard_hi,
                        int granule, int min_chunk, int target_units, int n_hb, void* ws, int max_units,
                        int max_split, int hq, int dv, int64_t* finish_ns, int* status, cudaStream_t s) {
    WsLayout lay = ws_layout(shard_hi - shard_lo, B, hq, dv, max_units, max_split);
    plan_kernel<<<1, kPlanThreads, 0, s>>>(seq_lens, B, N, I, q_len, shard_lo, shard_hi, granule, min_chunk,
                                           target_units, n_hb, reinterpret_cast<uint8_t*>(ws), lay, finish_ns, status);
    return cudaGetLastError();
}

}  // namespace dcp
