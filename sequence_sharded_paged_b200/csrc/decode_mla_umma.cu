// decode_mla_umma.cu -- split-KV MLA decode attention on 5th-generation tensor
// cores (tcgen05, accumulators in TMEM), bf16 latent cache or fp8 e4m3 latent
// cache with a per-token fp32 scale.
//
// Method: "Efficient Decode Context Parallelism with vLLM for Long Context
// Workloads", section 4.1 ("Compute": attention of the gathered query
// against the local KV slice, partial output + LSE) and section 5.3 (MLA:
// one 576-wide latent row per token shared by every query head; absorbed
// form: key = the whole row, value = its first 512 entries).
//
// Roofline: Hq = 64 heads do 2*64*(576 + 512) = 139k flop per latent row of
// 1152 bytes (bf16) or 580 bytes (fp8): 121 / 240 flop per byte, a dense
// contraction, so both products run on the tensor cores:
//   S   = Q . C^T   M = 64 heads (Q zero-padded to 64 rows), N = 32 tokens,
//                   K = 576; one thread per head row of S in TMEM, so the
//                   online softmax is thread-local;
//   O^T = V^T . P^T M = 128 value columns (four blocks of the 512), N = Hq,
//                   K = 32 tokens; V^T is read MN-major straight from the
//                   latent tile, P^T is written K-major by the softmax
//                   threads.  O^T occupies 4*Hq TMEM columns.
// The running maximum is rescaled lazily: O^T is rescaled only when a head's
// maximum grows by more than 2^8 (P then stays below 256).
//
// Tiles of 32 tokens (half a 64-token page): bf16 tiles (36 KB) arrive by
// TMA tiled loads (nine [32][64] boxes, 128-byte swizzle) into a 4-deep ring.
// fp8 tiles (18 KB + 128 B of scales) arrive by 1-D bulk copies into a 4-deep
// raw ring; four dequantising warps widen them to f16 (exact for every e4m3
// value) into a 2-deep ring of MMA tiles, and the MMAs run as kind::f16 with
// f16 operands.  The per-token scale multiplies the scores and P.
// P V always runs in f16 (P has 11 significant bits instead of bf16's 8): for a
// bf16 cache the softmax warps widen the tile's value columns to f16 in place
// once S has consumed them (values beyond +-65504 saturate).
//
// Warp roles (one CTA per SM, persistent, units taken from an atomic ticket):
//   warp 0      TMA / bulk-copy producer (lane 0)
//   warp 1      TMEM allocation, MMA issue (lane 0)
//   warps 2..5  softmax, lazy rescale of O^T, epilogue (one per TMEM lane quadrant)
//   warps 6..9  fp8 only: dequantisation
#include "common.cuh"
#include "finish.cuh"
#include "kernels.h"
#include "tma.h"
#include "umma.cuh"

namespace dcp {

namespace {

constexpr int kT = 32;                    // tokens per tile
constexpr int kKB = 9;                    // 576 = 9 blocks of 64 columns
constexpr int kBox = kT * 128;            // [32][64] 16-bit box with 128-byte rows
constexpr int kTileBytes = kKB * kBox;    // 36864
constexpr int kQBytes = kKB * 64 * 128;   // Q padded to 64 rows: 73728
constexpr int kPBytes = 64 * 64;          // P^T [64 heads][32 tokens] 16-bit, 64-byte rows
constexpr int kRawBytes = kT * 576;       // fp8 tile
constexpr int kNumTiles16 = 4;            // bf16: MMA tile ring depth
constexpr int kNumTilesF8 = 2;            // fp8: f16 MMA tile ring depth
constexpr int kNumRaw = 4;                // fp8: raw ring depth
constexpr float kRescaleLog2 = 8.f;       // lazy rescale threshold (log2 units)
constexpr int kSmBar = 1;                 // named barrier of the softmax warps

struct Smem {
    uint32_t q, tiles, p, raw, raw_scale, tile_scale, bars, meta, raw_meta, small, total;
};

template <bool FP8>
__host__ __device__ constexpr Smem smem_plan() {
    Smem s{};
    uint32_t o = 0;
    s.q = o;
    o += kQBytes;
    s.tiles = o;
    o += (FP8 ? kNumTilesF8 : kNumTiles16) * kTileBytes;
    s.p = o;
    o += 2 * kPBytes;
    s.raw = o;
    o += FP8 ? kNumRaw * kRawBytes : 0;
    s.raw_scale = o;
    o += FP8 ? kNumRaw * kT * 4 : 0;
    s.tile_scale = o;
    o += FP8 ? kNumTilesF8 * kT * 4 : 0;
    s.bars = o;
    o += 32 * 8;
    s.meta = o;
    o += 4 * 16;
    s.raw_meta = o;
    o += 4 * 16;
    s.small = o;  // m[64], l[64], alpha[64], misc[16]
    o += (3 * 64 + 16) * 4;
    s.total = o + 1024;  // alignment slack
    return s;
}

// barrier slots
enum : int {
    B_TILE_FULL = 0,    // [4]
    B_TILE_EMPTY = 4,   // [4]
    B_RAW_FULL = 8,     // [4]
    B_RAW_EMPTY = 12,   // [4]
    B_S_FULL = 16,      // [2]
    B_P_FULL = 18,      // [2]
    B_PV_DONE = 20,     // [2]
    B_Q_FULL = 22,
    B_Q_FREE = 23,
    B_O_FREE = 24,
    B_FINAL = 25,
};

__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
    return (uint32_t)(row * 128 + (((chunk ^ row) & 7) << 4));
}
__device__ __forceinline__ uint32_t sw64(int row, int chunk) {
    return (uint32_t)(row * 64 + (((chunk ^ (row >> 1)) & 3) << 4));
}

// OR of `pred` over the `nthreads` threads of named barrier `id` (all of them wait)
__device__ __forceinline__ int named_barrier_or(int id, int nthreads, int pred) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.s32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, %3, q;\n\t"
        "selp.s32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(pred), "r"(id), "r"(nthreads)
        : "memory");
    return r;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi, bool f16) {
    if (f16) {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    }
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

template <bool FP8, int HQ>
__global__ void __launch_bounds__(FP8 ? 320 : 192, 1)
    mla_umma_kernel(const __grid_constant__ CUtensorMap tmC, DecodeArgs a) {
    constexpr int NTILE = FP8 ? kNumTilesF8 : kNumTiles16;
    constexpr uint32_t FMT = FP8 ? 0u : 1u;  // f16 : bf16
    constexpr uint32_t IDESC_S = umma::idesc_f16(FMT, 0, 0, 64, kT);
    constexpr uint32_t IDESC_PV = umma::idesc_f16(0u, 1, 0, 128, HQ);  // P V always in f16
    constexpr Smem L = smem_plan<FP8>();

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L.bars);
    StageMeta* tmeta = reinterpret_cast<StageMeta*>(sm + L.meta);
    StageMeta* rmeta = reinterpret_cast<StageMeta*>(sm + L.raw_meta);
    float* s_m = reinterpret_cast<float*>(sm + L.small);
    float* s_l = s_m + 64;
    float* s_alpha = s_l + 64;
    int* s_misc = reinterpret_cast<int*>(s_alpha + 64);  // [0] tmem base, [1] any-rescale, [2] last flag
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_misc + 3);
    const float* tile_scale = reinterpret_cast<const float*>(sm + L.tile_scale);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sm_u32 = smem_u32(sm);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; i++) {
            mbar_init(bar + B_TILE_FULL + i, FP8 ? 4 : 1);
            mbar_init(bar + B_TILE_EMPTY + i, 1);
            mbar_init(bar + B_RAW_FULL + i, 1);
            mbar_init(bar + B_RAW_EMPTY + i, 4);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(bar + B_S_FULL + i, 1);
            mbar_init(bar + B_P_FULL + i, 4);
            mbar_init(bar + B_PV_DONE + i, 1);
        }
        mbar_init(bar + B_Q_FULL, 4);
        mbar_init(bar + B_Q_FREE, 1);
        mbar_init(bar + B_O_FREE, 4);
        mbar_init(bar + B_FINAL, 1);
        s_misc[1] = 0;
        *s_abort = 0;
        fence_barrier_init();
    }
    // Q rows >= HQ stay zero for the whole kernel
    for (int i = threadIdx.x; i < kQBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(sm + L.q)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (warp == 1) umma::tmem_alloc(reinterpret_cast<uint32_t*>(s_misc), 512);
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(s_misc);
    const uint32_t t_o = tmem;                  // O^T blocks: columns [blk*HQ, blk*HQ + HQ)
    const uint32_t t_s = tmem + 4 * HQ;         // S buffers: columns [4HQ + 32 sb, +32)
    const int num_units = a.plan->num_units;
    const int P = a.page_size;

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            if (!FP8) tma_prefetch_desc(&tmC);
            const int NS = FP8 ? kNumRaw : kNumTiles16;
            uint64_t* full = bar + (FP8 ? B_RAW_FULL : B_TILE_FULL);
            uint64_t* empty = bar + (FP8 ? B_RAW_EMPTY : B_TILE_EMPTY);
            StageMeta* meta = FP8 ? rmeta : tmeta;
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            while (ok) {
                const int ui = atomicAdd(a.ticket, 1);
                const bool done = ui >= num_units;
                Unit u;
                int nt = 1;
                if (!done) {
                    u = a.units[ui];
                    nt = (u.t1 - u.t0 + kT - 1) / kT;
                }
                int k = 0;
                do {
                    if (!mbar_wait(empty + stage, phase ^ 1, s_abort, a.status)) {
                        ok = false;
                        break;
                    }
                    if (done) {
                        meta[stage] = StageMeta{-1, 0, 0, 0};
                        mbar_arrive(full + stage);
                        ok = false;
                        break;
                    }
                    const int t = u.t0 + k * kT;
                    const int nvalid = nt == 0 ? 0 : min(u.t1 - t, kT);
                    const int flags = (k == 0 ? kStageFirst : 0) | (k >= nt - 1 ? kStageLast : 0);
                    int pg = -1;
                    if (nt > 0) {
                        pg = page_of(a, u.n, u.b, t / P);
                        if (pg < 0) record_status(a.status, DCP_ERR_UNALLOCATED_PAGE);
                    }
                    // flags bit 2 (kStageValid): data present; bits 8..15: valid token count
                    meta[stage] = StageMeta{ui, t, flags | (pg >= 0 ? kStageValid : 0) | ((pg >= 0 ? nvalid : 0) << 8),
                                            k};
                    if (pg >= 0) {
                        const int64_t row0 = (int64_t)pg * P + (t % P);
                        if (FP8) {
                            mbar_arrive_expect_tx(full + stage, kRawBytes + kT * 4);
                            bulk_g2s_hint(sm + L.raw + (size_t)stage * kRawBytes, a.k_pages + row0 * 576, kRawBytes,
                                          full + stage, pol);
                            bulk_g2s(sm + L.raw_scale + stage * kT * 4, a.kv_scales + row0, kT * 4, full + stage);
                        } else {
                            mbar_arrive_expect_tx(full + stage, kTileBytes);
                            uint8_t* dst = sm + L.tiles + (size_t)stage * kTileBytes;
#pragma unroll
                            for (int kb = 0; kb < kKB; kb++)
                                tma_load_2d(dst + kb * kBox, &tmC, kb * 64, (int32_t)row0, full + stage, pol);
                        }
                    } else {
                        mbar_arrive(full + stage);
                    }
                    issued++;
                    if (++stage == NS) {
                        stage = 0;
                        phase ^= 1;
                    }
                    k++;
                } while (k < nt);
            }
            if (*s_abort) {  // bounded drain of copies still in flight
                int n = issued < NS ? issued : NS;
                for (int i = 0; i < n; i++) {
                    stage = stage == 0 ? NS - 1 : stage - 1;
                    if (stage == NS - 1) phase ^= 1;
                    mbar_wait(full + stage, phase, nullptr, a.status);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int ts = 0;
            uint32_t tph = 0;
            uint32_t seq = 0, unit_k = 0, ofree_k = 0;
            bool pending = false;
            int pend_ts = 0, pend_sb = 0, pend_first = 0, pend_tokens = 0;
            uint32_t pend_seq = 0;
            bool ok = true;
            auto issue_pv = [&](void) -> bool {
                if (!mbar_wait(bar + B_P_FULL + pend_sb, (pend_seq >> 1) & 1, s_abort, a.status)) return false;
                if (pend_first) {
                    // epilogue of the previous unit has read O^T (first unit passes at once)
                    if (!mbar_wait(bar + B_O_FREE, (ofree_k & 1) ^ 1, s_abort, a.status)) return false;
                    ofree_k++;
                }
                umma::fence_after_sync();
                if (pend_tokens) {
                    const uint32_t tile = sm_u32 + L.tiles + (uint32_t)pend_ts * kTileBytes;
                    const uint32_t pbuf = sm_u32 + L.p + (uint32_t)pend_sb * kPBytes;
#pragma unroll
                    for (int blk = 0; blk < 4; blk++)
#pragma unroll
                        for (int ks = 0; ks < kT / 16; ks++) {
                            const uint64_t ad = umma::smem_desc(tile + (2 * blk) * kBox + ks * 2048, kBox, 1024,
                                                                umma::kSw128);
                            const uint64_t bd = umma::smem_desc(pbuf + ks * 32, 16, 512, umma::kSw64);
                            umma::mma_f16(t_o + blk * HQ, ad, bd, IDESC_PV, (pend_first && ks == 0) ? 0u : 1u);
                        }
                    umma::commit(bar + B_PV_DONE + pend_sb);
                    umma::commit(bar + B_TILE_EMPTY + pend_ts);
                } else {
                    mbar_arrive(bar + B_PV_DONE + pend_sb);
                    mbar_arrive(bar + B_TILE_EMPTY + pend_ts);
                }
                pending = false;
                return true;
            };
            while (ok) {
                if (!mbar_wait(bar + B_TILE_FULL + ts, tph, s_abort, a.status)) break;
                const StageMeta meta = load_meta(tmeta + ts);
                if (meta.unit < 0) break;
                const bool first = meta.flags & kStageFirst;
                const bool last = meta.flags & kStageLast;
                const bool tokens = true;  // S/PV run for every tile; masked tokens carry P = 0
                const int sb = seq & 1;
                if (first) {
                    if (pending && !issue_pv()) break;
                    if (!mbar_wait(bar + B_Q_FULL, unit_k & 1, s_abort, a.status)) break;
                    unit_k++;
                    umma::fence_after_sync();
                }
                {
                    const uint32_t tile = sm_u32 + L.tiles + (uint32_t)ts * kTileBytes;
                    const uint32_t qb = sm_u32 + L.q;
#pragma unroll
                    for (int kb = 0; kb < kKB; kb++)
#pragma unroll
                        for (int ks = 0; ks < 4; ks++) {
                            const uint64_t ad = umma::smem_desc(qb + kb * 8192 + ks * 32, 16, 1024, umma::kSw128);
                            const uint64_t bd = umma::smem_desc(tile + kb * kBox + ks * 32, 16, 1024, umma::kSw128);
                            umma::mma_f16(t_s + sb * kT, ad, bd, IDESC_S, (kb | ks) ? 1u : 0u);
                        }
                    umma::commit(bar + B_S_FULL + sb);
                }
                if (last) umma::commit(bar + B_Q_FREE);
                if (pending && !issue_pv()) break;
                pending = true;
                pend_ts = ts;
                pend_sb = sb;
                pend_first = first;
                pend_tokens = tokens;
                pend_seq = seq;
                seq++;
                if (++ts == NTILE) {
                    ts = 0;
                    tph ^= 1;
                }
            }
            if (pending && !*s_abort) issue_pv();
            // all MMAs complete before TMEM is released
            umma::commit(bar + B_FINAL);
            mbar_wait(bar + B_FINAL, 0, nullptr, a.status);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------------ softmax / epilogue
        // A failed (timed-out) wait sets `fail`; the four warps learn it at the
        // next named barrier of the group and leave the loop together, so no warp
        // is ever left waiting at a named barrier.
        const int qd = warp & 3;                 // TMEM lane quadrant
        const int h = 16 * qd + lane;            // head row of S owned by this thread (lane < 16)
        const bool head = lane < 16 && h < HQ;
        const int tid = threadIdx.x - 64;        // 0..127
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        int ts = 0;
        uint32_t tph = 0, seq = 0, unit_k = 0;
        float m_used = -INFINITY, lsum = 0.f;
        bool o_has = false;
        Unit u;
        u.n = u.b = u.t0 = u.t1 = u.slot = u.n_chunks = u.slot_base = u.pad = 0;
        bool fail = false;
        while (true) {
            if (!fail) fail = !mbar_wait(bar + B_TILE_FULL + ts, tph, s_abort, a.status);
            StageMeta meta{-1, 0, 0, 0};
            if (!fail) meta = load_meta(tmeta + ts);
            if (named_barrier_or(kSmBar, 128, fail)) break;
            if (meta.unit < 0) break;
            const bool first = meta.flags & kStageFirst;
            const bool last = meta.flags & kStageLast;
            const int nvalid = (meta.flags >> 8) & 0xFF;
            const int sb = seq & 1;
            if (first) {
                u = a.units[meta.unit];
                // Q of request u.b: all S MMAs of the previous unit are complete (first unit passes)
                fail = !mbar_wait(bar + B_Q_FREE, (unit_k & 1) ^ 1, s_abort, a.status);
                if (!fail) {
                    const uint4* qg = reinterpret_cast<const uint4*>(a.q + (int64_t)u.b * HQ * 576);
                    for (int i = tid; i < HQ * 72; i += 128) {
                        const int r = i / 72, c = i - r * 72;
                        uint4 v = __ldg(qg + i);
                        if (FP8) {
                            uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int e = 0; e < 4; e++) w[e] = pack2(bf16_lo(w[e]), bf16_hi(w[e]), true);
                            v = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                        *reinterpret_cast<uint4*>(sm + L.q + (c >> 3) * 8192 + sw128(r, c & 7)) = v;
                    }
                    umma::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar + B_Q_FULL);
                }
                unit_k++;
                m_used = -INFINITY;
                lsum = 0.f;
                o_has = false;
            }
            // ---- scores
            if (!fail) fail = !mbar_wait(bar + B_S_FULL + sb, (seq >> 1) & 1, s_abort, a.status);
            umma::fence_after_sync();
            uint32_t sr[32];
            umma::ld32(t_s + lane_off + sb * kT, sr);
            umma::wait_ld();
            float alpha = 1.f;
            float x[kT];
            if (head) {
                const float* tsc = tile_scale + ts * kT;
                float mt = -INFINITY;
#pragma unroll
                for (int j = 0; j < kT; j++) {
                    float v = __uint_as_float(sr[j]) * a.scale_log2;
                    if (FP8) v *= tsc[j];
                    x[j] = j < nvalid ? v : -INFINITY;
                    mt = fmaxf(mt, x[j]);
                }
                if (mt > m_used + kRescaleLog2 || (m_used == -INFINITY && mt != -INFINITY)) {
                    alpha = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - mt);
                    m_used = mt;
                }
                s_alpha[h] = alpha;
            }
            if (named_barrier_or(kSmBar, 128, fail)) break;
            // any head rescaled while O^T already holds data?
            const bool need = head && alpha != 1.f && o_has;
            const int any = named_barrier_or(kSmBar, 128, need);
            if (any) {
                // the previous tile's P V must be complete before O^T is touched
                fail = !mbar_wait(bar + B_PV_DONE + (sb ^ 1), ((seq - 1) >> 1) & 1, s_abort, a.status);
                if (!fail) {
                    umma::fence_after_sync();
#pragma unroll 1
                    for (int blk = 0; blk < 4; blk++) {
#pragma unroll 1
                        for (int c0 = 0; c0 < HQ; c0 += 16) {
                            uint32_t r[16];
                            umma::ld16(t_o + lane_off + blk * HQ + c0, r);
                            umma::wait_ld();
#pragma unroll
                            for (int i = 0; i < 16; i++)
                                r[i] = __float_as_uint(__uint_as_float(r[i]) * s_alpha[c0 + i]);
                            umma::st16(t_o + lane_off + blk * HQ + c0, r);
                        }
                    }
                    umma::wait_st();
                }
            }
            // ---- P^T row of this head (the P buffer is free once P V of tile seq-2 is complete)
            if (!fail) fail = !mbar_wait(bar + B_PV_DONE + sb, ((seq >> 1) & 1) ^ 1, s_abort, a.status);
            if (!fail && head) {
                const float* tsc = tile_scale + ts * kT;
                float rowsum = 0.f;
                uint32_t pw[kT / 2];
#pragma unroll
                for (int j = 0; j < kT; j += 2) {
                    // masked tokens (x = -inf) give 0, also while m_used is still -inf
                    float p0 = x[j] == -INFINITY ? 0.f : fast_exp2(x[j] - m_used);
                    float p1 = x[j + 1] == -INFINITY ? 0.f : fast_exp2(x[j + 1] - m_used);
                    rowsum += p0 + p1;
                    if (FP8) {
                        p0 *= tsc[j];
                        p1 *= tsc[j + 1];
                    }
                    pw[j / 2] = pack2(p0, p1, true);
                }
                lsum = lsum * alpha + rowsum;
                uint8_t* prow = sm + L.p + sb * kPBytes;
#pragma unroll
                for (int c = 0; c < 4; c++)
                    *reinterpret_cast<uint4*>(prow + sw64(h, c)) =
                        make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
            }
            if (!fail && !FP8) {
                // P V runs in f16 for both cache types: widen the tile's value columns (the
                // first 512, boxes 0..7) from bf16 to f16 in place now that S has read them,
                // saturating at +-65504; rows past the last valid token (stale page contents)
                // become zeros so that P = 0 cannot meet a NaN/Inf
                uint8_t* tile = sm + L.tiles + (size_t)ts * kTileBytes;
                for (int i = tid; i < 8 * kT * 8; i += 128) {
                    const int box = i / (kT * 8), rem = i - box * kT * 8;
                    const int r = rem >> 3;
                    uint4* ptr = reinterpret_cast<uint4*>(tile + box * kBox + r * 128 + (rem & 7) * 16);
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (r < nvalid) {
                        const uint4 w = *ptr;
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; e++)
                            o[e] = pack2(fminf(fmaxf(bf16_lo(ws[e]), -65504.f), 65504.f),
                                         fminf(fmaxf(bf16_hi(ws[e]), -65504.f), 65504.f), true);
                        v = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                    *ptr = v;
                }
            }
            umma::fence_proxy_async_smem();
            umma::fence_before_sync();
            __syncwarp();
            if (!fail && lane == 0) mbar_arrive(bar + B_P_FULL + sb);
            o_has = true;
            // ---- end of unit: O = O^T / l, LSE
            if (last) {
                if (!fail) fail = !mbar_wait(bar + B_PV_DONE + sb, (seq >> 1) & 1, s_abort, a.status);
                umma::fence_after_sync();
                if (head) {
                    s_m[h] = m_used;
                    s_l[h] = lsum;
                }
                if (named_barrier_or(kSmBar, 128, fail)) break;
                const int64_t shard = (int64_t)u.n * a.batch + u.b;
                const bool split = u.n_chunks > 1;
                float* obase = split ? a.split_o + (int64_t)u.slot * a.hq * 512 : a.o_partial + shard * a.hq * 512;
                float* lbase = split ? a.split_lse + (int64_t)u.slot * a.hq : a.lse + shard * a.hq;
#pragma unroll 1
                for (int blk = 0; blk < 4; blk++) {
                    const int dv = blk * 128 + 32 * qd + lane;
#pragma unroll 1
                    for (int c0 = 0; c0 < HQ; c0 += 16) {
                        uint32_t r[16];
                        umma::ld16(t_o + lane_off + blk * HQ + c0, r);
                        umma::wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; i++) {
                            const float l = s_l[c0 + i];
                            const float v = (l > 0.f) ? __uint_as_float(r[i]) / l : 0.f;
                            __stcg(obase + (int64_t)(c0 + i) * 512 + dv, v);
                        }
                    }
                }
                if (head) {
                    const float l = s_l[h];
                    __stcg(lbase + h, l > 0.f ? (s_m[h] + log2f(l)) * kLn2 : -INFINITY);
                }
                umma::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar + B_O_FREE);
                if (split) {
                    // split-KV reduce: the last chunk of the shard to finish merges the chunks
                    __threadfence();
                    named_barrier_sync(kSmBar, 128);
                    if (tid == 0) s_misc[2] = (atomicAdd(a.done + shard, 1) == u.n_chunks - 1) ? 1 : 0;
                    named_barrier_sync(kSmBar, 128);
                    const int is_last = *reinterpret_cast<volatile int*>(s_misc + 2);
                    named_barrier_sync(kSmBar, 128);
                    if (is_last) {
                        __threadfence();
                        const int K = u.n_chunks;
                        for (int i = tid; i < HQ * 128; i += 128) {
                            const int hh = i / 128, d4 = i % 128;
                            const float* lc = a.split_lse + (int64_t)u.slot_base * a.hq + hh;
                            float M = -INFINITY;
                            for (int j = 0; j < K; j++) M = fmaxf(M, __ldcg(lc + (int64_t)j * a.hq));
                            float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
                            float ws = 0.f;
                            if (M != -INFINITY) {
                                for (int j = 0; j < K; j++) {
                                    const float lj = __ldcg(lc + (int64_t)j * a.hq);
                                    if (lj == -INFINITY) continue;
                                    const float w = expf(lj - M);
                                    ws += w;
                                    const float4 xv = __ldcg(reinterpret_cast<const float4*>(
                                                                 a.split_o + ((int64_t)(u.slot_base + j) * a.hq + hh) * 512) +
                                                             d4);
                                    o.x += w * xv.x;
                                    o.y += w * xv.y;
                                    o.z += w * xv.z;
                                    o.w += w * xv.w;
                                }
                                const float inv = 1.f / ws;
                                o.x *= inv;
                                o.y *= inv;
                                o.z *= inv;
                                o.w *= inv;
                            }
                            reinterpret_cast<float4*>(a.o_partial + (shard * a.hq + hh) * 512)[d4] = o;
                            if (d4 == 0) a.lse[shard * a.hq + hh] = (M == -INFINITY) ? -INFINITY : M + logf(ws);
                        }
                    }
                }
            }
            seq++;
            if (++ts == NTILE) {
                ts = 0;
                tph ^= 1;
            }
        }
    } else if (FP8) {
        // ------------------------------------------------------------------ fp8 dequantisation
        const int tid = threadIdx.x - 192;  // 0..127
        int rs = 0, ts = 0;
        uint32_t rph = 0, tph = 0;
        while (true) {
            if (!mbar_wait(bar + B_RAW_FULL + rs, rph, s_abort, a.status)) break;
            const StageMeta meta = load_meta(rmeta + rs);
            if (!mbar_wait(bar + B_TILE_EMPTY + ts, tph ^ 1, s_abort, a.status)) break;
            if (meta.unit >= 0) {
                const int nvalid = (meta.flags >> 8) & 0xFF;
                const uint8_t* raw = sm + L.raw + (size_t)rs * kRawBytes;
                uint8_t* tile = sm + L.tiles + (size_t)ts * kTileBytes;
                for (int i = tid; i < kT * 72; i += 128) {
                    const int r = i / 72, c = i - r * 72;
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (r < nvalid) {
                        const uint2 w = *reinterpret_cast<const uint2*>(raw + r * 576 + c * 8);
                        __half2_raw h0 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w.x & 0xFFFF), __NV_E4M3);
                        __half2_raw h1 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w.x >> 16), __NV_E4M3);
                        __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w.y & 0xFFFF), __NV_E4M3);
                        __half2_raw h3 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w.y >> 16), __NV_E4M3);
                        v = make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                                       *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
                    }
                    *reinterpret_cast<uint4*>(tile + (c >> 3) * kBox + sw128(r, c & 7)) = v;
                }
                if (tid < kT) {
                    const float* rsc = reinterpret_cast<const float*>(sm + L.raw_scale) + rs * kT;
                    reinterpret_cast<float*>(sm + L.tile_scale)[ts * kT + tid] = tid < nvalid ? rsc[tid] : 0.f;
                }
            }
            if (tid == 0) tmeta[ts] = meta;
            umma::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar + B_TILE_FULL + ts);
                mbar_arrive(bar + B_RAW_EMPTY + rs);
            }
            if (meta.unit < 0) break;
            if (++rs == kNumRaw) {
                rs = 0;
                rph ^= 1;
            }
            if (++ts == NTILE) {
                ts = 0;
                tph ^= 1;
            }
        }
    }

    umma::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, 512);
    }
}

template <bool FP8, int HQ>
cudaError_t run(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s) {
    CUtensorMap tm;
    memset(&tm, 0, sizeof(tm));
    if (!FP8) {
        if (!make_tmap_2d(&tm, a.k_pages, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 576, (uint64_t)a.num_pages * a.page_size,
                          576 * 2, 64, kT, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    constexpr Smem L = smem_plan<FP8>();
    auto fn = mla_umma_kernel<FP8, HQ>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
    if (e != cudaSuccess) return e;
    fn<<<g.ctas, FP8 ? 320 : 192, L.total, s>>>(tm, a);
    return cudaGetLastError();
}

}  // namespace

bool mla_umma_supported(int hq, int page_size) { return (hq == 16 || hq == 32 || hq == 64) && page_size == 64; }

size_t mla_umma_smem_bytes(bool fp8) { return fp8 ? smem_plan<true>().total : smem_plan<false>().total; }

cudaError_t launch_decode_mla_umma(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s) {
    const bool fp8 = a.kv_scales != nullptr;
    switch (a.hq) {
        case 16: return fp8 ? run<true, 16>(g, a, s) : run<false, 16>(g, a, s);
        case 32: return fp8 ? run<true, 32>(g, a, s) : run<false, 32>(g, a, s);
        case 64: return fp8 ? run<true, 64>(g, a, s) : run<false, 64>(g, a, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace dcp
