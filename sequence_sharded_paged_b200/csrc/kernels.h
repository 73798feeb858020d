// kernels.h -- launch functions of the libdcp kernels (host-side declarations).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dcp.h"

namespace dcp {

struct DecodeArgs;

struct AppendArgs {
    int32_t kind, dtype;
    int32_t n_shards, interleave, page_size, num_pages, batch, max_local_pages;
    int32_t hkv, dk, dv;
    int64_t n_tok;
    const int32_t* req;
    const int32_t* pos;
    const uint8_t* k_new;
    const uint8_t* v_new;
    uint8_t* k_pages;
    uint8_t* v_pages;
    float* kv_scales;
    const int32_t* block_tables;
    int* status;
    int32_t only_shard;  // -1: block_tables holds every shard; r: only shard r's, rows of other shards are skipped
};

cudaError_t launch_shard_counts(int B, const int32_t* seq_lens, int N, int I, int32_t* counts, int* status,
                                cudaStream_t s);
cudaError_t launch_shard_map(int64_t n_pos, const int32_t* pos, const int32_t* req, int N, int I, int P,
                             const int32_t* bt, int B, int maxp, int num_pages, int32_t* rank_out,
                             int32_t* local_out, int64_t* slot_out, int* status, cudaStream_t s);
cudaError_t launch_append(const AppendArgs& a, cudaStream_t s);

// planner: splits every (shard, request) of shards [shard_lo, shard_hi) into
// chunks of at most chunk_tokens; output row block of shard n of request b:
// (n - shard_lo) * B + b
cudaError_t launch_plan(const int32_t* seq_lens, int B, int N, int I, int q_len, int shard_lo, int shard_hi,
                        int granule, int min_chunk, int target_units, int n_hb, void* ws, int max_units,
                        int max_split, int hq, int dv, int64_t* finish_ns, int* status, cudaStream_t s);

// decode kernels; each returns cudaErrorNotSupported for shapes it does not cover
enum class DecodePath { GqaSimt, GqaMma, MlaSimt, MlaUmma };
struct DecodeGeometry {
    DecodePath path;
    int n_hb;          // head blocks per unit (split counters are per (shard, head block))
    int ctas;          // persistent grid size
    int granule;       // chunk sizes are multiples of this many tokens
    int min_chunk;     // smallest chunk the planner makes
    int units_per_cta; // planner target
};
bool decode_geometry(int kind, int dtype, int hq, int hkv, int dk, int dv, int page_size, int num_sms,
                     DecodeGeometry* g);
cudaError_t launch_decode(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_decode_simt(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s);
size_t simt_smem_bytes(DecodePath p, int D, int G, int P, bool fp8);
int simt_blocks_per_sm(DecodePath p, int D, int G, int P, bool fp8);
bool gqa_mma_supported(int hq, int hkv, int dk);
int gqa_mma_blocks_per_sm(int hq, int hkv, int dk);
cudaError_t launch_decode_gqa_mma(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s);
// shapes the tensor-core MLA kernels take (both dtypes): Hq in {16, 32, 64}, 64-token pages
bool mla_umma_supported(int hq, int page_size);
cudaError_t launch_decode_mla_bf16(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_decode_mla_fp8(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s);

// discard != 0: o_partial is scratch whose lines are dropped from L2 once read
cudaError_t launch_merge(int N, int B, int H, int Dv, const float* o_partial, const float* lse, float* out,
                         float* lse_out, bool discard, cudaStream_t s);
cudaError_t launch_lse_rescale(int N, int rank, int B, int H, int Dv, const float* lse_all, const float* o,
                               float* o_rs, float* lse_out, cudaStream_t s);

}  // namespace dcp
