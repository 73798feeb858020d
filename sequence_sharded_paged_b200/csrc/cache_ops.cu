// cache_ops.cu -- shard map, per-shard counts and KV append (integer / copy work).
//
// Ownership follows the interleaved split of "Efficient Decode Context
// Parallelism with vLLM for Long Context Workloads", section 4 (each GPU holds
// the KV of a subset of positions) with the granularity of the "Decode
// Context Parallel Guide"'s cp_kv_cache_interleave_size: p -> shard
// (p / I) mod N, local index (p / (I N)) * I + p mod I.
#include "common.cuh"
#include "kernels.h"

namespace dcp {

__global__ void shard_counts_kernel(int B, const int32_t* __restrict__ seq_lens, int N, int I,
                                    int32_t* __restrict__ counts, int* status) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= N * B) return;
    int n = i / B, b = i - n * B;
    int64_t L = seq_lens[b];
    if (L < 0) {
        record_status(status, DCP_ERR_INVALID_ARG);
        L = 0;
    }
    counts[i] = (int32_t)count_of(L, N, I, n);
}

__global__ void shard_map_kernel(int64_t n_pos, const int32_t* __restrict__ pos, const int32_t* __restrict__ req,
                                 int N, int I, int P, const int32_t* __restrict__ bt, int B, int maxp, int num_pages,
                                 int32_t* __restrict__ rank_out, int32_t* __restrict__ local_out,
                                 int64_t* __restrict__ slot_out, int* status) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_pos) return;
    int64_t p = pos[i];
    int b = req ? req[i] : (int)i;
    if (p < 0) {
        record_status(status, DCP_ERR_INVALID_ARG);
        rank_out[i] = -1;
        local_out[i] = -1;
        slot_out[i] = -1;
        return;
    }
    int r = owner_of(p, N, I);
    int64_t l = local_of(p, N, I);
    rank_out[i] = r;
    local_out[i] = (int32_t)l;
    int64_t j = l / P;
    int pg = -1;
    if (b >= 0 && b < B && j < maxp) pg = bt[((int64_t)r * B + b) * maxp + j];
    if (pg < 0 || pg >= num_pages) {
        record_status(status, DCP_ERR_UNALLOCATED_PAGE);
        slot_out[i] = -1;
    } else {
        slot_out[i] = (int64_t)pg * P + l % P;
    }
}

// Resolve (req, pos) -> physical page and in-page offset; -1 page when invalid,
// -2 when another rank owns the position (rank-local cache).
__device__ __forceinline__ int append_target(const AppendArgs& a, int64_t i, int* off) {
    int64_t p = a.pos[i];
    int b = a.req ? a.req[i] : (int)i;
    if (p < 0 || b < 0 || b >= a.batch) return -1;
    int r = owner_of(p, a.n_shards, a.interleave);
    if (a.only_shard >= 0) {
        if (r != a.only_shard) return -2;
        r = 0;  // the rank's tables are row 0
    }
    int64_t l = local_of(p, a.n_shards, a.interleave);
    int64_t j = l / a.page_size;
    if (j >= a.max_local_pages) return -1;
    int pg = a.block_tables[((int64_t)r * a.batch + b) * a.max_local_pages + j];
    if (pg < 0 || pg >= a.num_pages) return -1;
    *off = (int)(l % a.page_size);
    return pg;
}

// GQA: one warp per (token, kv head): copy the K and V rows (16-byte vectors).
__global__ void append_gqa_kernel(AppendArgs a) {
    int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    if (w >= a.n_tok * a.hkv) return;
    int64_t i = w / a.hkv;
    int g = (int)(w - i * a.hkv);
    int off = 0;
    int pg = append_target(a, i, &off);
    if (pg < 0) {
        if (pg == -1 && lane == 0) record_status(a.status, DCP_ERR_UNALLOCATED_PAGE);
        return;
    }
    const int P = a.page_size;
    {
        const uint4* src = reinterpret_cast<const uint4*>(a.k_new + ((i * a.hkv + g) * a.dk) * 2);
        uint4* dst = reinterpret_cast<uint4*>(a.k_pages + ((((int64_t)pg * a.hkv + g) * P + off) * a.dk) * 2);
        for (int v = lane; v < a.dk / 8; v += 32) dst[v] = src[v];
    }
    {
        const uint4* src = reinterpret_cast<const uint4*>(a.v_new + ((i * a.hkv + g) * a.dv) * 2);
        uint4* dst = reinterpret_cast<uint4*>(a.v_pages + ((((int64_t)pg * a.hkv + g) * P + off) * a.dv) * 2);
        for (int v = lane; v < a.dv / 8; v += 32) dst[v] = src[v];
    }
}

// MLA bf16: one warp per token: copy the 576-wide latent row.
__global__ void append_mla_bf16_kernel(AppendArgs a) {
    int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    if (i >= a.n_tok) return;
    int off = 0;
    int pg = append_target(a, i, &off);
    if (pg < 0) {
        if (pg == -1 && lane == 0) record_status(a.status, DCP_ERR_UNALLOCATED_PAGE);
        return;
    }
    const uint4* src = reinterpret_cast<const uint4*>(a.k_new + i * a.dk * 2);
    uint4* dst = reinterpret_cast<uint4*>(a.k_pages + (((int64_t)pg * a.page_size + off) * a.dk) * 2);
    for (int v = lane; v < a.dk / 8; v += 32) dst[v] = src[v];
}

// MLA fp8: one warp per token: amax over the row, scale = amax / 448 (fp32,
// round to nearest), code = RNE(x / scale) saturated to +-448.
__global__ void append_mla_fp8_kernel(AppendArgs a) {
    int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    if (i >= a.n_tok) return;
    int off = 0;
    int pg = append_target(a, i, &off);
    if (pg < 0) {
        if (pg == -1 && lane == 0) record_status(a.status, DCP_ERR_UNALLOCATED_PAGE);
        return;
    }
    // 576 bf16 = 72 chunks of 8; lane owns chunks lane, lane+32, lane+64 (< 72)
    const uint4* src = reinterpret_cast<const uint4*>(a.k_new + i * a.dk * 2);
    const int nch = a.dk / 8;
    uint4 c[3];
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 3; k++) {
        int ch = lane + 32 * k;
        if (ch < nch) {
            c[k] = src[ch];
            uint32_t w[4] = {c[k].x, c[k].y, c[k].z, c[k].w};
#pragma unroll
            for (int e = 0; e < 4; e++) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[e])), fabsf(bf16_hi(w[e]))));
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float scale = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
    uint8_t* dst = a.k_pages + ((int64_t)pg * a.page_size + off) * a.dk;
#pragma unroll
    for (int k = 0; k < 3; k++) {
        int ch = lane + 32 * k;
        if (ch < nch) {
            uint32_t w[4] = {c[k].x, c[k].y, c[k].z, c[k].w};
            uint32_t packed[2] = {0, 0};
#pragma unroll
            for (int e = 0; e < 4; e++) {
                float x0 = amax == 0.f ? 0.f : __fdiv_rn(bf16_lo(w[e]), scale);
                float x1 = amax == 0.f ? 0.f : __fdiv_rn(bf16_hi(w[e]), scale);
                uint32_t b0 = __nv_cvt_float_to_fp8(x0, __NV_SATFINITE, __NV_E4M3);
                uint32_t b1 = __nv_cvt_float_to_fp8(x1, __NV_SATFINITE, __NV_E4M3);
                packed[e >> 1] |= (b0 | (b1 << 8)) << (16 * (e & 1));
            }
            *reinterpret_cast<uint2*>(dst + ch * 8) = make_uint2(packed[0], packed[1]);
        }
    }
    if (lane == 0) a.kv_scales[(int64_t)pg * a.page_size + off] = scale;
}

static int blocks_for(int64_t threads, int per_block) {
    int64_t g = (threads + per_block - 1) / per_block;
    return (int)(g < 1 ? 1 : g);
}

cudaError_t launch_shard_counts(int B, const int32_t* seq_lens, int N, int I, int32_t* counts, int* status,
                                cudaStream_t s) {
    shard_counts_kernel<<<blocks_for((int64_t)N * B, 256), 256, 0, s>>>(B, seq_lens, N, I, counts, status);
    return cudaGetLastError();
}

cudaError_t launch_shard_map(int64_t n_pos, const int32_t* pos, const int32_t* req, int N, int I, int P,
                             const int32_t* bt, int B, int maxp, int num_pages, int32_t* rank_out,
                             int32_t* local_out, int64_t* slot_out, int* status, cudaStream_t s) {
    if (n_pos == 0) return cudaSuccess;
    shard_map_kernel<<<blocks_for(n_pos, 256), 256, 0, s>>>(n_pos, pos, req, N, I, P, bt, B, maxp, num_pages,
                                                            rank_out, local_out, slot_out, status);
    return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t s) {
    if (a.n_tok == 0) return cudaSuccess;
    if (a.kind == DCP_GQA) {
        append_gqa_kernel<<<blocks_for(a.n_tok * a.hkv * 32, 256), 256, 0, s>>>(a);
    } else if (a.dtype == DCP_BF16) {
        append_mla_bf16_kernel<<<blocks_for(a.n_tok * 32, 256), 256, 0, s>>>(a);
    } else {
        append_mla_fp8_kernel<<<blocks_for(a.n_tok * 32, 256), 256, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace dcp
