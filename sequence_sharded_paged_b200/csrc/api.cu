// api.cu -- the C ABI of libdcp (include/dcp.h): host-side validation, the
// sticky device status word, workspace sizing and kernel dispatch.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace dcp {

// In selftest.cu; declared here rather than in kernels.h because only this entry point calls it.
cudaError_t launch_selftest_bounded_wait(int* status, int64_t* result, cudaStream_t s);

// Sticky status word, one per device context.
static __device__ int g_status;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;

// The addresses of this library's __device__ arrays belong to the CUDA context
// that loaded the module: a context rebuilt after cudaDeviceReset reloads it
// elsewhere.  So they are cached per device together with the id of the
// context they were looked up in, and looked up again when that id changes.
struct DeviceCache {
    unsigned long long ctx_id = 0;
    bool valid = false;
    int* status = nullptr;
    uint8_t* scratch = nullptr;  // built-in decode scratch, looked up on first use
    int num_sms = 0;
};
DeviceCache g_dev[kMaxDevices];

using PFN_ctxGetCurrent = CUresult (*)(CUcontext*);
using PFN_ctxGetId = CUresult (*)(CUcontext, unsigned long long*);
std::once_flag g_ctx_once;
PFN_ctxGetCurrent g_ctx_get_current = nullptr;
PFN_ctxGetId g_ctx_get_id = nullptr;

void load_ctx_entries() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_ctx_get_current = reinterpret_cast<PFN_ctxGetCurrent>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_ctx_get_id = reinterpret_cast<PFN_ctxGetId>(fn);
}

// Id of the calling thread's current context (0 when none is current or the
// driver cannot say).
unsigned long long current_ctx_id() {
    std::call_once(g_ctx_once, load_ctx_entries);
    if (!g_ctx_get_current || !g_ctx_get_id) return 0;
    CUcontext ctx = nullptr;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    if (g_ctx_get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

dcp_status cuda_err(cudaError_t e) { return e == cudaSuccess ? DCP_OK : DCP_ERR_CUDA; }

// The cache entry of the current device, valid for its current context.  Must
// be called with g_mu held.
dcp_status device_entry(DeviceCache** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DCP_ERR_CUDA;
    DeviceCache& d = g_dev[dev];
    unsigned long long id = current_ctx_id();
    if (!d.valid || id == 0 || id != d.ctx_id) {
        // cudaGetSymbolAddress makes the device's primary context current when
        // none is, so the id is read again after it
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return DCP_ERR_CUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DCP_ERR_CUDA;
        d.status = static_cast<int*>(p);
        d.scratch = nullptr;
        d.num_sms = sms;
        d.ctx_id = current_ctx_id();
        d.valid = true;
    }
    *out = &d;
    return DCP_OK;
}

// device address of g_status and SM count of the current device
dcp_status device_info(int** status, int* num_sms) {
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceCache* d = nullptr;
    dcp_status st = device_entry(&d);
    if (st != DCP_OK) return st;
    if (status) *status = d->status;
    if (num_sms) *num_sms = d->num_sms;
    return DCP_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape/descriptor checks shared by every call that takes a cache.
dcp_status check_desc(const dcp_cache_desc* c, bool need_pools) {
    if (!c) return DCP_ERR_INVALID_ARG;
    if (c->n_shards < 1 || c->interleave < 1 || c->num_pages < 1 || c->batch < 1 || c->max_local_pages < 1)
        return DCP_ERR_INVALID_ARG;
    if (c->page_size != 16 && c->page_size != 64) return DCP_ERR_UNSUPPORTED;
    if ((int64_t)c->max_local_pages * c->page_size > ((int64_t)1 << 31) - 1) return DCP_ERR_INVALID_ARG;
    if (!c->block_tables) return DCP_ERR_INVALID_ARG;
    if (c->hq < 1 || c->hkv < 1 || c->hq % c->hkv) return DCP_ERR_INVALID_ARG;
    if (c->kind == DCP_GQA) {
        if (c->dtype != DCP_BF16) return DCP_ERR_UNSUPPORTED;
        if (c->dk != c->dv || (c->dk != 64 && c->dk != 128)) return DCP_ERR_UNSUPPORTED;
        if (need_pools && (!c->k_pages || !c->v_pages)) return DCP_ERR_INVALID_ARG;
        if (need_pools && (!aligned16(c->k_pages) || !aligned16(c->v_pages))) return DCP_ERR_MISALIGNED;
    } else if (c->kind == DCP_MLA) {
        if (c->hkv != 1 || c->dk != 576 || c->dv != 512) return DCP_ERR_UNSUPPORTED;
        if (c->hq % 16) return DCP_ERR_UNSUPPORTED;
        if (c->dtype != DCP_BF16 && c->dtype != DCP_FP8_E4M3) return DCP_ERR_INVALID_ARG;
        if (need_pools && !c->k_pages) return DCP_ERR_INVALID_ARG;
        if (need_pools && c->dtype == DCP_FP8_E4M3 && !c->kv_scales) return DCP_ERR_INVALID_ARG;
        if (need_pools && (!aligned16(c->k_pages) || (c->kv_scales && !aligned16(c->kv_scales))))
            return DCP_ERR_MISALIGNED;
    } else {
        return DCP_ERR_INVALID_ARG;
    }
    if (!aligned16(c->block_tables)) return DCP_ERR_MISALIGNED;
    return DCP_OK;
}

// What a decode call produces (dcp_decode_mode): every shard's partial (the
// caller's o_partial / lse), the merged output (per-shard partials in the
// workspace, then the LSE merge), or one rank's shard of a multi-GPU group.
enum PlanMode { kModePartial = DCP_DECODE_PARTIAL, kModeMerged = DCP_DECODE_MERGED, kModeRank = DCP_DECODE_RANK };

struct Plan {
    DecodeGeometry g;
    WsLayout lay;
    size_t off_qs = 0, off_qinv = 0;  // fp8 MLA query split (0 when unused)
    size_t off_part = 0, off_part_lse = 0;  // merged mode: the per-shard partials
    int q_len = 1;                    // query tokens per request (rows = q_len * hq)
    int mode = kModePartial;
};

constexpr int kMaxQueryLen = 64;

// The fp8 MLA kernel reads the query split into two e4m3 terms from the end of
// the workspace: [B][128 rows][576] bytes + [B][64] fp32 reciprocals.
void add_query_split(const dcp_cache_desc* c, int B, Plan* p) {
    p->off_qs = p->off_qinv = 0;
    if (p->g.path != DecodePath::MlaUmma || c->dtype != DCP_FP8_E4M3) return;
    p->off_qs = p->lay.total;
    p->off_qinv = align256(p->off_qs + (size_t)B * 128 * 576);
    p->lay.total = align256(p->off_qinv + (size_t)B * 64 * sizeof(float));
}

// The plan of a decode of B requests with q_len query tokens each (q_len * hq
// query rows) in the given mode.  Several query tokens are served by the
// tensor-core paths only.  Split slots are needed only for shards longer than
// one chunk: at most 2 * target + 2 of them.
bool make_plan(const dcp_cache_desc* c, int B, int q_len, int mode, int num_sms, Plan* p) {
    if (q_len < 1 || q_len > kMaxQueryLen || mode < kModePartial || mode > kModeRank) return false;
    const int rows = q_len * c->hq;
    if (!decode_geometry(c->kind, c->dtype, rows, c->hkv, c->dk, c->dv, c->page_size, num_sms, &p->g)) return false;
    if (q_len > 1 && p->g.path != DecodePath::GqaMma && p->g.path != DecodePath::MlaUmma) return false;
    const int shards = mode == kModeRank ? 1 : c->n_shards;
    const int64_t target = (int64_t)p->g.units_per_cta * p->g.ctas;
    const int64_t max_units = (int64_t)shards * B + target + 1;
    const int64_t max_split = 2 * target + 2;
    if (max_units > (1 << 30)) return false;
    p->lay = ws_layout(shards, B, rows, c->dv, (int)max_units, (int)max_split);
    p->q_len = q_len;
    p->mode = mode;
    add_query_split(c, B, p);
    p->off_part = p->off_part_lse = 0;
    if (mode == kModeMerged) {
        p->off_part = p->lay.total;
        p->off_part_lse = align256(p->off_part + sizeof(float) * (size_t)shards * B * rows * c->dv);
        p->lay.total = align256(p->off_part_lse + sizeof(float) * (size_t)shards * B * rows);
    }
    return true;
}

// ---------------------------------------------------------------------------
// built-in decode scratch (dcp_decode_partial_noalloc)
// ---------------------------------------------------------------------------
// One per device context.  Its address is looked up on the first no-alloc call
// in a context (and again if the context is rebuilt), with that device current.
static __device__ __align__(256) uint8_t g_decode_scratch[DCP_STATIC_SCRATCH_BYTES];

dcp_status decode_scratch(uint8_t** out) {
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceCache* d = nullptr;
    dcp_status st = device_entry(&d);
    if (st != DCP_OK) return st;
    if (!d->scratch) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return DCP_ERR_CUDA;
        d->scratch = static_cast<uint8_t*>(p);
    }
    *out = d->scratch;
    return DCP_OK;
}

// make_plan's plan when its workspace fits in `cap` bytes; otherwise the same
// geometry with half the units per CTA (a smaller chunk target, hence fewer
// split slots), repeated down to one unit per CTA.  The bounds are make_plan's
// for the smaller target.  False when nothing fits.
bool make_plan_within(const dcp_cache_desc* c, int B, int num_sms, size_t cap, Plan* p) {
    if (!make_plan(c, B, 1, kModePartial, num_sms, p)) return false;
    while (p->lay.total > cap && p->g.units_per_cta > 1) {
        p->g.units_per_cta /= 2;
        const int64_t target = (int64_t)p->g.units_per_cta * p->g.ctas;
        const int64_t max_units = (int64_t)c->n_shards * B + target + 1;
        p->lay = ws_layout(c->n_shards, B, c->hq, c->dv, (int)max_units, (int)(2 * target + 2));
        add_query_split(c, B, p);
    }
    return p->lay.total <= cap;
}

// The launch sequence of the decode (plan kernel, decode kernel) on a workspace
// `w` laid out by `p`.
// rank >= 0: the cache holds only shard `rank`'s block tables, and only that
// shard is decoded.
dcp_status decode_on(const dcp_cache_desc* cache, int32_t B, const void* q, const int32_t* seq_lens,
                     float* o_partial, float* lse, uint8_t* w, const Plan& p, int* status, cudaStream_t s,
                     int64_t* finish_ns = nullptr, int rank = -1) {
    const int64_t target = (int64_t)p.g.units_per_cta * p.g.ctas;
    const int rows = p.q_len * cache->hq;
    const int shard_lo = rank >= 0 ? rank : 0, shard_hi = rank >= 0 ? rank + 1 : cache->n_shards;
    cudaError_t e = launch_plan(seq_lens, B, cache->n_shards, cache->interleave, p.q_len, shard_lo, shard_hi,
                                p.g.granule, p.g.min_chunk, (int)target, p.g.n_hb, w, p.lay.max_units,
                                p.lay.max_split, rows, cache->dv, finish_ns, status, s);
    if (e != cudaSuccess) return DCP_ERR_CUDA;
    DecodeArgs a;
    a.k_pages = static_cast<const uint8_t*>(cache->k_pages);
    a.v_pages = static_cast<const uint8_t*>(cache->v_pages);
    a.kv_scales = cache->dtype == DCP_FP8_E4M3 ? cache->kv_scales : nullptr;
    a.block_tables = cache->block_tables;
    a.n_shards = cache->n_shards;
    a.interleave = cache->interleave;
    a.page_size = cache->page_size;
    a.num_pages = cache->num_pages;
    a.batch = B;
    a.max_local_pages = cache->max_local_pages;
    a.hq = rows;
    a.hkv = cache->hkv;
    a.dk = cache->dk;
    a.dv = cache->dv;
    a.scale_log2 = cache->scale * kLog2e;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.seq_lens = seq_lens;
    a.o_partial = o_partial;
    a.lse = lse;
    a.plan = reinterpret_cast<const PlanHeader*>(w);
    a.ticket = &reinterpret_cast<PlanHeader*>(w)->next_unit;
    a.units = reinterpret_cast<const Unit*>(w + p.lay.off_units);
    a.done = reinterpret_cast<int32_t*>(w + p.lay.off_done);
    a.split_o = reinterpret_cast<float*>(w + p.lay.off_split_o);
    a.split_lse = reinterpret_cast<float*>(w + p.lay.off_split_lse);
    a.qs = p.off_qs ? w + p.off_qs : nullptr;
    a.qinv = p.off_qinv ? reinterpret_cast<float*>(w + p.off_qinv) : nullptr;
    a.status = status;
    a.q_len = p.q_len;
    a.finish_ns = finish_ns;
    a.bt_shard0 = rank >= 0 ? rank : 0;
    e = launch_decode(p.g, a, s);
    if (e == cudaErrorNotSupported) return DCP_ERR_UNSUPPORTED;
    return cuda_err(e);
}

}  // namespace

// ---------------------------------------------------------------------------
// decode dispatch
// ---------------------------------------------------------------------------
bool decode_geometry(int kind, int dtype, int hq, int hkv, int dk, int dv, int page_size, int num_sms,
                     DecodeGeometry* g) {
    (void)dv;
    if (kind == DCP_GQA && gqa_mma_supported(hq, hkv, dk)) {
        const int occ = gqa_mma_blocks_per_sm(hq, hkv, dk);
        if (occ < 1) return false;
        g->path = DecodePath::GqaMma;
        g->n_hb = 1;
        g->ctas = num_sms * occ;
        g->granule = page_size;
        g->min_chunk = 1024;
        g->units_per_cta = 16;
        return true;
    }
    if (kind == DCP_GQA) {
        const int G = hq / hkv;
        if (G != 1 && G != 2 && G != 4 && G != 8) return false;
        const int occ = simt_blocks_per_sm(DecodePath::GqaSimt, dk, G, page_size, false);
        if (occ < 1) return false;
        g->path = DecodePath::GqaSimt;
        g->n_hb = hkv;
        g->ctas = num_sms * occ;
        g->granule = page_size;
        g->min_chunk = 512;
        g->units_per_cta = 4;
        return true;
    }
    if (kind == DCP_MLA && mla_umma_supported(hq, page_size)) {
        g->path = DecodePath::MlaUmma;
        g->n_hb = 1;
        g->ctas = num_sms;  // one CTA per SM (shared memory and the whole TMEM)
        g->granule = page_size;
        g->min_chunk = 2048;
        // fewer, longer chunks: every chunk boundary costs an epilogue and a split merge here
        g->units_per_cta = 8;
        return true;
    }
    if (kind == DCP_MLA) {
        const int occ = simt_blocks_per_sm(DecodePath::MlaSimt, dk, hq, page_size, dtype == DCP_FP8_E4M3);
        if (occ < 1) return false;
        g->path = DecodePath::MlaSimt;
        g->n_hb = hq / 16;
        g->ctas = num_sms * occ;
        g->granule = page_size;
        g->min_chunk = 1024;
        g->units_per_cta = 4;
        return true;
    }
    return false;
}

bool mla_umma_supported(int hq, int page_size) { return (hq == 16 || hq == 32 || hq == 64) && page_size == 64; }

cudaError_t launch_decode(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s) {
    switch (g.path) {
        case DecodePath::GqaSimt:
        case DecodePath::MlaSimt:
            return launch_decode_simt(g, a, s);
        case DecodePath::GqaMma:
            return launch_decode_gqa_mma(g, a, s);
        case DecodePath::MlaUmma:
            return a.kv_scales ? launch_decode_mla_fp8(g, a, s) : launch_decode_mla_bf16(g, a, s);
        default:
            return cudaErrorNotSupported;
    }
}

}  // namespace dcp

using namespace dcp;

extern "C" {

const char* dcp_status_string(dcp_status s) {
    switch (s) {
        case DCP_OK: return "ok";
        case DCP_ERR_INVALID_ARG: return "invalid argument";
        case DCP_ERR_UNSUPPORTED: return "unsupported shape";
        case DCP_ERR_UNALLOCATED_PAGE: return "unallocated page";
        case DCP_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case DCP_ERR_CUDA: return "CUDA error";
        case DCP_ERR_MISALIGNED: return "misaligned pointer";
        case DCP_ERR_TIMEOUT: return "kernel wait timed out";
    }
    return "unknown status";
}

dcp_status dcp_shard_counts(int32_t B, const int32_t* seq_lens, int32_t N, int32_t I, int32_t* counts_out,
                            void* stream) {
    if (B < 1 || N < 1 || I < 1 || !seq_lens || !counts_out) return DCP_ERR_INVALID_ARG;
    int* status = nullptr;
    dcp_status st = device_info(&status, nullptr);
    if (st != DCP_OK) return st;
    return cuda_err(launch_shard_counts(B, seq_lens, N, I, counts_out, status, (cudaStream_t)stream));
}

dcp_status dcp_shard_map(const dcp_cache_desc* cache, int64_t n_pos, const int32_t* pos, const int32_t* req,
                         int32_t* rank_out, int32_t* local_out, int64_t* slot_out, void* stream) {
    dcp_status st = check_desc(cache, false);
    if (st != DCP_OK) return st;
    if (n_pos < 0) return DCP_ERR_INVALID_ARG;
    if (n_pos == 0) return DCP_OK;
    if (!pos || !rank_out || !local_out || !slot_out) return DCP_ERR_INVALID_ARG;
    int* status = nullptr;
    st = device_info(&status, nullptr);
    if (st != DCP_OK) return st;
    return cuda_err(launch_shard_map(n_pos, pos, req, cache->n_shards, cache->interleave, cache->page_size,
                                     cache->block_tables, cache->batch, cache->max_local_pages, cache->num_pages,
                                     rank_out, local_out, slot_out, status, (cudaStream_t)stream));
}

static dcp_status kv_append(const dcp_cache_desc* cache, int32_t only_shard, int64_t n_tok, const int32_t* req,
                            const int32_t* pos, const void* k_new, const void* v_new, void* stream) {
    dcp_status st = check_desc(cache, true);
    if (st != DCP_OK) return st;
    if (n_tok < 0) return DCP_ERR_INVALID_ARG;
    if (n_tok == 0) return DCP_OK;
    if (!pos || !k_new || (cache->kind == DCP_GQA && !v_new)) return DCP_ERR_INVALID_ARG;
    if (!aligned16(k_new) || (v_new && !aligned16(v_new))) return DCP_ERR_MISALIGNED;
    int* status = nullptr;
    st = device_info(&status, nullptr);
    if (st != DCP_OK) return st;
    AppendArgs a;
    a.kind = cache->kind;
    a.dtype = cache->dtype;
    a.n_shards = cache->n_shards;
    a.interleave = cache->interleave;
    a.page_size = cache->page_size;
    a.num_pages = cache->num_pages;
    a.batch = cache->batch;
    a.max_local_pages = cache->max_local_pages;
    a.hkv = cache->hkv;
    a.dk = cache->dk;
    a.dv = cache->dv;
    a.n_tok = n_tok;
    a.req = req;
    a.pos = pos;
    a.k_new = static_cast<const uint8_t*>(k_new);
    a.v_new = static_cast<const uint8_t*>(v_new);
    a.k_pages = static_cast<uint8_t*>(cache->k_pages);
    a.v_pages = static_cast<uint8_t*>(cache->v_pages);
    a.kv_scales = cache->kv_scales;
    a.block_tables = cache->block_tables;
    a.status = status;
    a.only_shard = only_shard;
    return cuda_err(launch_append(a, (cudaStream_t)stream));
}

dcp_status dcp_kv_append(const dcp_cache_desc* cache, int64_t n_tok, const int32_t* req, const int32_t* pos,
                         const void* k_new, const void* v_new, void* stream) {
    return kv_append(cache, -1, n_tok, req, pos, k_new, v_new, stream);
}

dcp_status dcp_kv_append_rank(const dcp_cache_desc* cache, int32_t rank, int64_t n_tok, const int32_t* req,
                              const int32_t* pos, const void* k_new, const void* v_new, void* stream) {
    if (!cache || rank < 0 || rank >= cache->n_shards) return DCP_ERR_INVALID_ARG;
    return kv_append(cache, rank, n_tok, req, pos, k_new, v_new, stream);
}

size_t dcp_decode_workspace_size(const dcp_cache_desc* cache, int32_t B) {
    if (check_desc(cache, false) != DCP_OK || B != cache->batch) return 0;
    int num_sms = 0;
    if (device_info(nullptr, &num_sms) != DCP_OK) return 0;
    Plan p;
    if (!make_plan(cache, B, 1, kModePartial, num_sms, &p)) return 0;
    return p.lay.total;
}

size_t dcp_decode_workspace_size_ex(const dcp_cache_desc* cache, int32_t B, int32_t q_len, int32_t mode) {
    if (check_desc(cache, false) != DCP_OK || B != cache->batch) return 0;
    int num_sms = 0;
    if (device_info(nullptr, &num_sms) != DCP_OK) return 0;
    Plan p;
    if (!make_plan(cache, B, q_len, mode, num_sms, &p)) return 0;
    return p.lay.total;
}

dcp_status dcp_decode_partial(const dcp_cache_desc* cache, int32_t B, const void* q, const int32_t* seq_lens,
                              float* o_partial, float* lse, void* ws, size_t ws_bytes, void* stream) {
    dcp_status st = check_desc(cache, true);
    if (st != DCP_OK) return st;
    if (B != cache->batch || !q || !seq_lens || !o_partial || !lse || !ws) return DCP_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o_partial) || !aligned16(lse) || !aligned16(ws)) return DCP_ERR_MISALIGNED;
    int* status = nullptr;
    int num_sms = 0;
    st = device_info(&status, &num_sms);
    if (st != DCP_OK) return st;
    Plan p;
    if (!make_plan(cache, B, 1, kModePartial, num_sms, &p)) return DCP_ERR_UNSUPPORTED;
    if (ws_bytes < p.lay.total) return DCP_ERR_WORKSPACE_TOO_SMALL;
    return decode_on(cache, B, q, seq_lens, o_partial, lse, static_cast<uint8_t*>(ws), p, status, (cudaStream_t)stream);
}

// Shared checks and launch of the decode calls that take a query length
// (rank >= 0: only that shard, from a cache holding only its tables).
static dcp_status decode_ex(const dcp_cache_desc* cache, int32_t B, int32_t q_len, int mode, const void* q,
                            const int32_t* seq_lens, float* out, float* lse, int64_t* finish_ns, void* ws,
                            size_t ws_bytes, void* stream, int rank = -1) {
    dcp_status st = check_desc(cache, true);
    if (st != DCP_OK) return st;
    if (rank >= cache->n_shards) return DCP_ERR_INVALID_ARG;
    if (B != cache->batch || q_len < 1 || !q || !seq_lens || !out || !lse || !ws) return DCP_ERR_INVALID_ARG;
    if (q_len > kMaxQueryLen) return DCP_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(out) || !aligned16(lse) || !aligned16(ws) || (finish_ns && !aligned16(finish_ns)))
        return DCP_ERR_MISALIGNED;
    int* status = nullptr;
    int num_sms = 0;
    st = device_info(&status, &num_sms);
    if (st != DCP_OK) return st;
    Plan p;
    if (!make_plan(cache, B, q_len, mode, num_sms, &p)) return DCP_ERR_UNSUPPORTED;
    if (ws_bytes < p.lay.total) return DCP_ERR_WORKSPACE_TOO_SMALL;
    uint8_t* w = static_cast<uint8_t*>(ws);
    if (mode != kModeMerged)
        return decode_on(cache, B, q, seq_lens, out, lse, w, p, status, (cudaStream_t)stream, finish_ns, rank);
    // merged output: every shard's partial into the workspace, then the LSE merge; the
    // kernel boundary orders the partials' stores before the merge reads them, and the
    // merge drops the partials' lines from L2 once read
    const int rows = q_len * cache->hq;
    float* part = reinterpret_cast<float*>(w + p.off_part);
    float* part_lse = reinterpret_cast<float*>(w + p.off_part_lse);
    st = decode_on(cache, B, q, seq_lens, part, part_lse, w, p, status, (cudaStream_t)stream, finish_ns);
    if (st != DCP_OK) return st;
    return cuda_err(launch_merge(cache->n_shards, B, rows, cache->dv, part, part_lse, out, lse, true,
                                 (cudaStream_t)stream));
}

dcp_status dcp_decode_partial_multi(const dcp_cache_desc* cache, int32_t B, int32_t q_len, const void* q,
                                    const int32_t* seq_lens, float* o_partial, float* lse, void* ws, size_t ws_bytes,
                                    void* stream) {
    return decode_ex(cache, B, q_len, kModePartial, q, seq_lens, o_partial, lse, nullptr, ws, ws_bytes, stream);
}

dcp_status dcp_decode_merged(const dcp_cache_desc* cache, int32_t B, int32_t q_len, const void* q,
                             const int32_t* seq_lens, float* out, float* lse_out, int64_t* finish_ns, void* ws,
                             size_t ws_bytes, void* stream) {
    return decode_ex(cache, B, q_len, kModeMerged, q, seq_lens, out, lse_out, finish_ns, ws, ws_bytes, stream);
}

dcp_status dcp_decode_rank(const dcp_cache_desc* cache, int32_t rank, int32_t B, int32_t q_len, const void* q,
                           const int32_t* seq_lens, float* o, float* lse, void* ws, size_t ws_bytes, void* stream) {
    if (!cache || rank < 0) return DCP_ERR_INVALID_ARG;
    return decode_ex(cache, B, q_len, kModeRank, q, seq_lens, o, lse, nullptr, ws, ws_bytes, stream, rank);
}

// No workspace argument and no allocation: for callers that cannot allocate
// device memory where they decode (a serving process whose caching allocator
// holds the free HBM for its KV pool; loops that cannot take cudaMalloc's
// implicit synchronisation).  One scratch array per device: overlapping calls
// race on it.
dcp_status dcp_decode_partial_noalloc(const dcp_cache_desc* cache, int32_t B, const void* q,
                                      const int32_t* seq_lens, float* o_partial, float* lse, void* stream) {
    dcp_status st = check_desc(cache, true);
    if (st != DCP_OK) return st;
    if (B != cache->batch || !q || !seq_lens || !o_partial || !lse) return DCP_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o_partial) || !aligned16(lse)) return DCP_ERR_MISALIGNED;
    int* status = nullptr;
    int num_sms = 0;
    st = device_info(&status, &num_sms);
    if (st != DCP_OK) return st;
    Plan p;
    if (!make_plan(cache, B, 1, kModePartial, num_sms, &p)) return DCP_ERR_UNSUPPORTED;
    if (!make_plan_within(cache, B, num_sms, DCP_STATIC_SCRATCH_BYTES, &p)) return DCP_ERR_WORKSPACE_TOO_SMALL;
    uint8_t* w = nullptr;
    st = decode_scratch(&w);
    if (st != DCP_OK) return st;
    return decode_on(cache, B, q, seq_lens, o_partial, lse, w, p, status, (cudaStream_t)stream);
}

dcp_status dcp_merge(int32_t N, int32_t B, int32_t H, int32_t Dv, const float* o_partial, const float* lse,
                     float* out, float* lse_out, void* stream) {
    if (N < 1 || B < 1 || H < 1 || Dv < 4 || Dv % 4 || !o_partial || !lse || !out) return DCP_ERR_INVALID_ARG;
    if (!aligned16(o_partial) || !aligned16(out)) return DCP_ERR_MISALIGNED;
    return cuda_err(launch_merge(N, B, H, Dv, o_partial, lse, out, lse_out, false, (cudaStream_t)stream));
}

dcp_status dcp_lse_rescale(int32_t N, int32_t rank, int32_t B, int32_t H, int32_t Dv, const float* lse_all,
                           const float* o, float* o_rs, float* lse_out, void* stream) {
    if (N < 1 || rank < 0 || rank >= N || B < 1 || H < 1 || H % N || Dv < 4 || Dv % 4 || !lse_all || !o || !o_rs)
        return DCP_ERR_INVALID_ARG;
    if (!aligned16(o) || !aligned16(o_rs)) return DCP_ERR_MISALIGNED;
    return cuda_err(launch_lse_rescale(N, rank, B, H, Dv, lse_all, o, o_rs, lse_out, (cudaStream_t)stream));
}

dcp_status dcp_selftest_bounded_wait(int64_t* result, void* stream) {
    if (!result) return DCP_ERR_INVALID_ARG;
    if (!aligned16(result)) return DCP_ERR_MISALIGNED;
    int* status = nullptr;
    dcp_status st = device_info(&status, nullptr);
    if (st != DCP_OK) return st;
    return cuda_err(launch_selftest_bounded_wait(status, result, (cudaStream_t)stream));
}

dcp_status dcp_get_device_status(int32_t* status_out, void* stream) {
    if (!status_out) return DCP_ERR_INVALID_ARG;
    int* status = nullptr;
    dcp_status st = device_info(&status, nullptr);
    if (st != DCP_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaStreamSynchronize(s) != cudaSuccess) return DCP_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return DCP_ERR_CUDA;
    if (cudaMemset(status, 0, sizeof(int)) != cudaSuccess) return DCP_ERR_CUDA;
    *status_out = v;
    return DCP_OK;
}

}  // extern "C"
