// decode_mla_bf16.cu -- split-KV MLA decode attention over a bf16 latent cache
// on 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// Method: "Efficient Decode Context Parallelism with vLLM for Long Context
// Workloads", section 4.1 ("Compute": attention of the gathered query against
// the local KV slice, partial output + LSE) and section 5.3 (MLA: one 576-wide
// latent row per token shared by every query head; absorbed form: key = the
// whole row, value = its first 512 entries).
//
// Per 64-token tile (one page; 72 KB):
//   S   = Q . C^T   bf16, M = 64 heads (Q zero-padded), N = 64 tokens, K = 576:
//                   36 MMAs; one thread per head row of S, so the online
//                   softmax is thread-local;
//   O^T = V^T . P^T bf16, M = 128 value columns (four blocks of the 512),
//                   N = Hq, K = 64 tokens, twice: P is split exactly into
//                   P_hi = bf16(p) and P_lo = bf16(p - P_hi) (residual below
//                   2^-16 relative), so P keeps ~16 significant bits with
//                   bf16 operands and V^T is read MN-major straight from the
//                   tile: 32 MMAs.
// Measured tcgen05 cost on this part is >= ~46 cycles per MMA instruction, so
// tiles are as wide as shared memory allows: Q (72 KB) + two 72 KB tiles.
// P_hi^T goes into the tile's rope box, which S no longer needs; P_lo^T into
// one extra 8 KB buffer.  Rows past the last valid token carry P = 0 and their
// value columns are zeroed, so stale page contents cannot meet P.  The running
// maximum is rescaled lazily: O^T is rescaled only when a head's maximum grows
// by more than 2^8 (P then stays below 256).
//
// Warp roles (224 threads, one CTA per SM, persistent, units taken from an
// atomic ticket):
//   warp 0      TMA producer: nine [64][64] boxes per tile, 128 B swizzle
//   warp 1      TMEM allocation; lane 0 issues the S MMAs of each tile
//   warps 2..5  softmax, lazy rescale of O^T, epilogue (one per TMEM lane
//               quadrant; lanes l and l + 16 share head l's 64 tokens)
//   warp 6      lane 0 issues the P V MMAs of each tile
#include "common.cuh"
#include "finish.cuh"
#include "kernels.h"
#include "tma.h"
#include "umma.cuh"

namespace dcp {

// Optional timeline of CTA 0 (SM clock at each protocol step), compiled only
// with -DDCP_TRACE for profiling builds; expands to nothing otherwise.
#ifdef DCP_TRACE
__device__ unsigned long long g_mla_trace[16][512];
#define TRACE(ev, k)                                                          \
    do {                                                                      \
        if (blockIdx.x == 0 && (k) < 512) g_mla_trace[ev][(k)] = clock64();   \
    } while (0)
extern "C" int dcp_trace_read(unsigned long long* host) {
    return (int)cudaMemcpyFromSymbol(host, g_mla_trace, sizeof(g_mla_trace));
}
#else
#define TRACE(ev, k) \
    do {             \
    } while (0)
#endif

namespace {

constexpr int kT = 64;                    // tokens per tile (one page)
constexpr int kKB = 9;                    // 576 = 9 blocks of 64 columns
constexpr int kBox = kT * 128;            // [64][64] 16-bit box with 128-byte rows: 8 KB
constexpr int kTileBytes = kKB * kBox;    // 73728
constexpr int kQBytes = kKB * 64 * 128;   // Q padded to 64 rows: 73728
constexpr int kStages = 2;
constexpr float kRescaleLog2 = 8.f;
constexpr int kSmBar = 1;                 // named barrier of the softmax warps
constexpr int kThreads = 224;              // producer, S issuer, softmax x 4, P V issuer
constexpr int kPBytes = 64 * 128;         // P_lo^T [64 heads][64 tokens] bf16

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffTiles = kQBytes;
constexpr uint32_t kOffPlo = kOffTiles + kStages * kTileBytes;
constexpr uint32_t kOffBars = kOffPlo + kPBytes;
constexpr uint32_t kOffMeta = kOffBars + 32 * 8;
constexpr uint32_t kOffSmall = kOffMeta + kStages * 16;
constexpr uint32_t kSmemBytes = kOffSmall + (3 * 64 + 16) * 4 + 1024;

enum : int {
    B_TILE_FULL = 0,   // [2]
    B_TILE_EMPTY = 2,  // [2]
    B_S_FULL = 4,      // [2]
    B_P_FULL = 6,      // [2]
    B_PV_DONE = 10,    // [2]
    B_Q_FULL = 12,
    B_Q_FREE = 13,
    B_O_FREE = 14,
    B_FINAL = 15,
};

__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
    return (uint32_t)(row * 128 + (((chunk ^ row) & 7) << 4));
}

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

template <int HQ>
__global__ void __launch_bounds__(kThreads, 1)
    mla_bf16_kernel(const __grid_constant__ CUtensorMap tmC, DecodeArgs a) {
    constexpr uint32_t IDESC_S = umma::idesc_f16(1u, 0, 0, 64, kT);      // bf16, K-major A and B
    constexpr uint32_t IDESC_PV = umma::idesc_f16(1u, 1, 0, 128, HQ);    // bf16, V^T MN-major, P^T K-major

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kOffBars);
    StageMeta* tmeta = reinterpret_cast<StageMeta*>(sm + kOffMeta);
    float* s_m = reinterpret_cast<float*>(sm + kOffSmall);
    float* s_l = s_m + 64;
    float* s_alpha = s_l + 64;
    int* s_misc = reinterpret_cast<int*>(s_alpha + 64);  // [0] tmem base, [2] split flag, [3] abort
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_misc + 3);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sm_u32 = smem_u32(sm);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; i++) {
            mbar_init(bar + B_TILE_FULL + i, 1);
            mbar_init(bar + B_TILE_EMPTY + i, 1);
            mbar_init(bar + B_S_FULL + i, 1);
            mbar_init(bar + B_P_FULL + i, 4);
            mbar_init(bar + B_PV_DONE + i, 1);
        }
        mbar_init(bar + B_Q_FULL, 4);
        mbar_init(bar + B_Q_FREE, 1);
        mbar_init(bar + B_O_FREE, 4);
        mbar_init(bar + B_FINAL, 2);
        *s_abort = 0;
        fence_barrier_init();
    }
    // Q rows >= HQ stay zero for the whole kernel
    for (int i = threadIdx.x; i < kQBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(sm + kOffQ)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (warp == 1) umma::tmem_alloc(reinterpret_cast<uint32_t*>(s_misc), 512);
    umma::fence_proxy_async_smem();
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(s_misc);
    const uint32_t t_o = tmem;              // O^T: columns [blk*HQ, blk*HQ + HQ)
    const uint32_t t_s = tmem + 4 * HQ;     // S buffers: [4HQ + 64 sb, +64)
    const int num_units = a.plan->num_units;
    const int P = a.page_size;

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        // Nothing between a free stage and its tile's copies waits on global memory: the next
        // unit (ticket, record, and the first 64 of its block-table entries) is fetched before
        // the current one ends, and each lane holds one entry of the current 32-tile
        // window of the unit, the following window loaded 32 tiles ahead.  Lanes 0..8 issue
        // the tile's nine boxes at once.
        const uint64_t pol = l2_policy_evict_first();
        if (lane == 0) tma_prefetch_desc(&tmC);
        struct Cursor {
            int ui;      // unit index
            Unit u;
            int np;      // tiles with tokens (0 for an empty unit, which still yields one tile)
            int w0, w1;  // this lane's block-table entry of the current / next 32-tile window
        };
        // block-table entry of tile i of unit c (-1 past its tiles or its table row)
        auto entry = [&](const Cursor& c, int i) -> int { return i < c.np ? page_of(a, c.u.n, c.u.b, c.u.t0 / P + i) : -1; };
        auto fetch = [&](Cursor& c) -> bool {
            int t = 0;
            if (lane == 0) t = atomicAdd(a.ticket, 1);
            c.ui = __shfl_sync(0xffffffffu, t, 0);
            if (c.ui >= num_units) return false;
            c.u = a.units[c.ui];
            c.np = (c.u.t1 - c.u.t0 + kT - 1) / kT;
            c.w0 = entry(c, lane);
            c.w1 = entry(c, 32 + lane);
            return true;
        };
        // the next unit is fetched 2 tiles before the current one ends (early enough to hide
        // the ticket -> record -> entries chain, late enough not to hold a unit another CTA
        // could start)
        constexpr int kAhead = 2;
        Cursor cur, nxt;
        bool have = fetch(cur);
        bool fetched = false, have_nxt = false;
        int k = 0, stage = 0, issued = 0;
        uint32_t phase = 0;
        while (true) {
            int waited = 1;
            if (lane == 0) waited = mbar_wait(bar + B_TILE_EMPTY + stage, phase ^ 1, s_abort, a.status);
            if (!__shfl_sync(0xffffffffu, waited, 0)) break;
            if (lane == 0) TRACE(14, issued);
            if (!have) {
                if (lane == 0) {
                    tmeta[stage] = StageMeta{-1, 0, 0, 0};
                    mbar_arrive(bar + B_TILE_FULL + stage);
                }
                break;
            }
            const int nt = max(1, cur.np);
            const int t = cur.u.t0 + k * kT;
            const int pg = __shfl_sync(0xffffffffu, cur.w0, k & 31);
            const int nvalid = cur.np == 0 ? 0 : min(cur.u.t1 - t, kT);
            const int flags = (k == 0 ? kStageFirst : 0) | (k == nt - 1 ? kStageLast : 0);
            if (lane == 0) {
                if (cur.np > 0 && pg < 0) record_status(a.status, DCP_ERR_UNALLOCATED_PAGE);
                tmeta[stage] = StageMeta{cur.ui, t, flags | ((pg >= 0 ? nvalid : 0) << 8), k};
            }
            if (pg >= 0) {
                if (lane == 0) mbar_arrive_expect_tx(bar + B_TILE_FULL + stage, kTileBytes);
                __syncwarp();
                if (lane < kKB)
                    tma_load_2d(sm + kOffTiles + (size_t)stage * kTileBytes + lane * kBox, &tmC, lane * 64, pg * P,
                                bar + B_TILE_FULL + stage, pol);
            } else if (lane == 0) {
                mbar_arrive(bar + B_TILE_FULL + stage);
            }
            if (lane == 0) TRACE(15, issued);
            issued++;
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1;
            }
            // next tile: the next window of this unit, or the unit fetched ahead
            ++k;
            if (!fetched && nt - k <= kAhead) {
                have_nxt = fetch(nxt);
                fetched = true;
            }
            if (k < nt) {
                if ((k & 31) == 0) {
                    cur.w0 = cur.w1;
                    cur.w1 = entry(cur, k + 32 + lane);
                }
            } else {
                have = have_nxt;
                fetched = false;
                k = 0;
                if (have) cur = nxt;
            }
        }
        if (lane == 0 && *s_abort) {  // bounded drain of copies still in flight
            int n = issued < kStages ? issued : kStages;
            for (int i = 0; i < n; i++) {
                stage = stage == 0 ? kStages - 1 : stage - 1;
                if (stage == kStages - 1) phase ^= 1;
                mbar_wait(bar + B_TILE_FULL + stage, phase, nullptr, a.status);
            }
        }
    } else if (warp == 1 || warp == 6) {
        // ------------------------------------------------------------------ MMA issuers
        // Two threads.  Warp 1 issues S of each tile once it has landed, the softmax has read
        // the S buffer's previous tile (its P is ready) and (first tile of a unit) Q is loaded.
        // Warp 6 issues P V of each tile once its P is ready; its completion frees the tile for
        // the next load.  Each thread's waits hide behind the other's MMAs.
        if (lane == 0) {
            const uint64_t dt0 = umma::smem_desc(sm_u32 + kOffTiles, 16, 1024, umma::kSw128);
            uint32_t unit_k = 0, ofree_k = 0;
            if (warp == 1) {
                const uint64_t dq0 = umma::smem_desc(sm_u32 + kOffQ, 16, 1024, umma::kSw128);
                for (uint32_t k = 0;; k++) {
                    const int ts = k & 1;
                    if (!mbar_wait(bar + B_TILE_FULL + ts, (k >> 1) & 1, s_abort, a.status)) break;
                    const StageMeta meta = load_meta(tmeta + ts);
                    if (meta.unit < 0) break;
                    if (k >= 2 && !mbar_wait(bar + B_P_FULL + ts, ((k - 2) >> 1) & 1, s_abort, a.status)) break;
                    const bool first = meta.flags & kStageFirst;
                    if (first) {
                        if (!mbar_wait(bar + B_Q_FULL, unit_k & 1, s_abort, a.status)) break;
                        unit_k++;
                    }
                    TRACE(0, k);
                    umma::fence_after_sync();
                    const uint64_t tile = (uint64_t)((ts * kTileBytes) >> 4);
#pragma unroll
                    for (int kb = 0; kb < kKB; kb++)
#pragma unroll
                        for (int ks = 0; ks < 4; ks++) {
                            const uint64_t off = (uint64_t)((kb * kBox + ks * 32) >> 4);
                            umma::mma_f16(t_s + ts * kT, dq0 + off, dt0 + tile + off, IDESC_S, (kb | ks) ? 1u : 0u);
                        }
                    umma::commit(bar + B_S_FULL + ts);
                    if (meta.flags & kStageLast) umma::commit(bar + B_Q_FREE);
                    TRACE(1, k);
                }
            } else {
                const uint64_t dv0 = umma::smem_desc(sm_u32 + kOffTiles, kBox, 1024, umma::kSw128);
                for (uint32_t k = 0;; k++) {
                    const int sb = k & 1;
                    // the tile's metadata stays in place until this thread frees the tile
                    if (!mbar_wait(bar + B_TILE_FULL + sb, (k >> 1) & 1, s_abort, a.status)) break;
                    const StageMeta meta = load_meta(tmeta + sb);
                    if (meta.unit < 0) break;
                    if (!mbar_wait(bar + B_P_FULL + sb, (k >> 1) & 1, s_abort, a.status)) break;
                    const bool fst = meta.flags & kStageFirst;
                    if (fst) {
                        if (!mbar_wait(bar + B_O_FREE, (ofree_k & 1) ^ 1, s_abort, a.status)) break;
                        ofree_k++;
                    }
                    TRACE(2, k);
                    umma::fence_after_sync();
                    const uint64_t tile = (uint64_t)((sb * kTileBytes) >> 4);
                    // P_hi^T sits in the tile's rope box, P_lo^T in its own buffer; consecutive
                    // MMAs go to different accumulator blocks
                    const uint64_t phi = dt0 + tile + (uint64_t)((8 * kBox) >> 4);
                    const uint64_t plo = dt0 + (uint64_t)((kOffPlo - kOffTiles) >> 4);
#pragma unroll
                    for (int ks = 0; ks < kT / 16; ks++)
#pragma unroll
                        for (int term = 0; term < 2; term++)
#pragma unroll
                            for (int blk = 0; blk < 4; blk++) {
                                const uint64_t ad = dv0 + tile + (uint64_t)(((2 * blk) * kBox + ks * 2048) >> 4);
                                umma::mma_f16(t_o + blk * HQ, ad, (term ? plo : phi) + (uint64_t)(ks * 2), IDESC_PV,
                                              (fst && ks == 0 && term == 0) ? 0u : 1u);
                            }
                    umma::commit(bar + B_PV_DONE + sb);
                    umma::commit(bar + B_TILE_EMPTY + sb);
                    TRACE(4, k);
                }
            }
            umma::commit(bar + B_FINAL);
            mbar_wait(bar + B_FINAL, 0, nullptr, a.status);
        }
    } else {
        // ------------------------------------------------------------------ softmax / epilogue
        // A failed (timed-out) wait sets `fail`; the four warps learn it at the
        // next named barrier of the group and leave the loop together.
        // S rows live in lanes 0..15 of each TMEM quadrant (M = 64 layout); lane l + 16 takes
        // tokens 32..63 of the head of lane l, received by shuffles.
        const int qd = warp & 3;                 // TMEM lane quadrant
        const int half = lane >> 4;              // 0: tokens 0..31 of the tile, 1: tokens 32..63
        const int h = 16 * qd + (lane & 15);     // head
        const bool head = h < HQ;
        const int base = 32 * half;
        const int tid = threadIdx.x - 64;        // 0..127
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        uint32_t seq = 0, unit_k = 0;
        float m_used = -INFINITY, lsum = 0.f;
        int lim = 0x7fffffff;  // local tokens [0, lim) of the unit's shard this row attends
        bool o_has = false;
        bool fail = false;
        Unit u{};
        while (true) {
            const int ts = seq & 1;
            const uint32_t par = (seq >> 1) & 1;
            if (!fail) fail = !mbar_wait(bar + B_TILE_FULL + ts, par, s_abort, a.status);
            if (threadIdx.x == 64) TRACE(5, seq);
            StageMeta meta{-1, 0, 0, 0};
            if (!fail) meta = load_meta(tmeta + ts);
            if (named_barrier_or(kSmBar, 128, fail)) break;
            if (meta.unit < 0) break;
            const bool first = meta.flags & kStageFirst;
            const bool last = meta.flags & kStageLast;
            const int nvalid = (meta.flags >> 8) & 0xFF;
            if (first) {
                u = a.units[meta.unit];
                lim = head ? row_limit(a, u, h / (HQ / a.q_len)) : 0x7fffffff;
                // Q of request u.b: all S MMAs of the previous unit are complete (first unit passes)
                fail = !mbar_wait(bar + B_Q_FREE, (unit_k & 1) ^ 1, s_abort, a.status);
                if (!fail) {
                    const uint4* qg = reinterpret_cast<const uint4*>(a.q + (int64_t)u.b * HQ * 576);
                    for (int i = tid; i < HQ * 72; i += 128) {
                        const int r = i / 72, c = i - r * 72;
                        *reinterpret_cast<uint4*>(sm + kOffQ + (c >> 3) * 8192 + sw128(r, c & 7)) = __ldg(qg + i);
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
            if (!fail) fail = !mbar_wait(bar + B_S_FULL + ts, par, s_abort, a.status);
            if (threadIdx.x == 64) TRACE(6, seq);
            umma::fence_after_sync();
            // tokens of the tile this row attends: the tile's valid tokens, cut by the row's
            // causal limit when the request has several query tokens
            const int row_nv = min(nvalid, max(0, lim - meta.t));
            float x[32];
            {
                uint32_t v0[32], v1[32];
                umma::ld32(t_s + lane_off + ts * kT, v0);
                umma::ld32(t_s + lane_off + ts * kT + 32, v1);
                umma::wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j++) {
                    const uint32_t recv = __shfl_xor_sync(0xffffffffu, v1[j], 16);
                    const float v = __uint_as_float(half ? recv : v0[j]);
                    x[j] = base + j < row_nv ? v * a.scale_log2 : -INFINITY;
                }
            }
            float mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; j++) mt = fmaxf(mt, x[j]);
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
            float alpha = 1.f;
            if (mt > m_used + kRescaleLog2 || (m_used == -INFINITY && mt != -INFINITY)) {
                alpha = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - mt);
                m_used = mt;
            }
            if (head && half == 0) s_alpha[h] = alpha;
            if (threadIdx.x == 64) TRACE(7, seq);
            // one barrier: some head rescaled while O^T holds data, or a wait failed (a failing
            // thread republishes the abort flag first, so every thread reads it set after the barrier)
            if (fail) *s_abort = 1;
            const int any = named_barrier_or(kSmBar, 128, fail || (head && alpha != 1.f && o_has));
            if (threadIdx.x == 64) TRACE(8, seq);
            if (any && *s_abort) break;
            // the previous tile's P V must be complete before O^T is rescaled or the
            // P_lo buffer rewritten (the first tile of the kernel passes at once)
            // (seq = 0: (seq - 1) wraps, giving parity 1, which a fresh barrier reports complete)
            if (!fail) fail = !mbar_wait(bar + B_PV_DONE + (ts ^ 1), ((seq - 1) >> 1) & 1, s_abort, a.status);
            if (any && !fail) {
                umma::fence_after_sync();
#pragma unroll 1
                for (int blk = 0; blk < 4; blk++) {
#pragma unroll 1
                    for (int c0 = 0; c0 < HQ; c0 += 16) {
                        uint32_t r[16];
                        umma::ld16(t_o + lane_off + blk * HQ + c0, r);
                        umma::wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; i++) r[i] = __float_as_uint(__uint_as_float(r[i]) * s_alpha[c0 + i]);
                        umma::st16(t_o + lane_off + blk * HQ + c0, r);
                    }
                }
                umma::wait_st();
            }
            // ---- P^T row of this head: P_hi into the tile's rope box (dead once S has
            // read it), P_lo into its buffer
            if (!fail && head) {
                float rowsum = 0.f;
                uint32_t phw[16], plw[16];
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float x0 = x[j], x1 = x[j + 1];
                    const float p0 = x0 == -INFINITY ? 0.f : fast_exp2(x0 - m_used);
                    const float p1 = x1 == -INFINITY ? 0.f : fast_exp2(x1 - m_used);
                    rowsum += p0 + p1;
                    const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
                    const float2 hf = __bfloat1622float2(hi);
                    const __nv_bfloat162 lo = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
                    phw[j / 2] = *reinterpret_cast<const uint32_t*>(&hi);
                    plw[j / 2] = *reinterpret_cast<const uint32_t*>(&lo);
                }
                lsum = lsum * alpha + rowsum;
                uint8_t* prow = sm + kOffTiles + (size_t)ts * kTileBytes + 8 * kBox;
                uint8_t* lrow = sm + kOffPlo;
                // my 32 tokens = 16-byte chunks 4 half .. 4 half + 3 of row h
#pragma unroll
                for (int cc = 0; cc < 4; cc++) {
                    const int c = 4 * half + cc;
                    *reinterpret_cast<uint4*>(prow + sw128(h, c)) =
                        make_uint4(phw[4 * cc], phw[4 * cc + 1], phw[4 * cc + 2], phw[4 * cc + 3]);
                    *reinterpret_cast<uint4*>(lrow + sw128(h, c)) =
                        make_uint4(plw[4 * cc], plw[4 * cc + 1], plw[4 * cc + 2], plw[4 * cc + 3]);
                }
            }
            if (!fail && nvalid < kT) {
                // rows past the last valid token hold stale page contents: zero their value
                // columns so that P = 0 cannot meet a NaN/Inf
                uint8_t* tile = sm + kOffTiles + (size_t)ts * kTileBytes;
                const int nr = kT - nvalid;
                for (int i = tid; i < nr * 8 * 8; i += 128) {
                    const int box = i / (nr * 8), rem = i - box * nr * 8;
                    const int r = nvalid + rem / 8, c = rem & 7;
                    *reinterpret_cast<uint4*>(tile + box * kBox + r * 128 + c * 16) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            if (threadIdx.x == 64) TRACE(9, seq);
            umma::fence_proxy_async_smem();
            umma::fence_before_sync();
            __syncwarp();
            if (!fail && lane == 0) mbar_arrive(bar + B_P_FULL + ts);
            if (threadIdx.x == 64) TRACE(10, seq);
            o_has = true;
            // ---- end of unit: O = O^T / l, LSE
            if (last) {
                if (!fail) fail = !mbar_wait(bar + B_PV_DONE + ts, par, s_abort, a.status);
                umma::fence_after_sync();
                const float l = lsum + __shfl_xor_sync(0xffffffffu, lsum, 16);  // both halves of the head
                if (head && half == 0) s_l[h] = l > 0.f ? 1.f / l : 0.f;      // O = O^T * (1 / l)
                if (named_barrier_or(kSmBar, 128, fail)) break;
                const int64_t grp = u.grp;
                const bool split = u.n_chunks > 1;
                float* obase = split ? a.split_o + (int64_t)u.slot * a.hq * 512 : a.o_partial + grp * a.hq * 512;
                float* lbase = split ? a.split_lse + (int64_t)u.slot * a.hq : a.lse + grp * a.hq;
#pragma unroll 1
                for (int blk = 0; blk < 4; blk++) {
                    const int dv = blk * 128 + 32 * qd + lane;
#pragma unroll 1
                    for (int c0 = 0; c0 < HQ; c0 += 16) {
                        uint32_t r[16];
                        umma::ld16(t_o + lane_off + blk * HQ + c0, r);
                        umma::wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; i++)
                            __stcg(obase + (int64_t)(c0 + i) * 512 + dv, __uint_as_float(r[i]) * s_l[c0 + i]);
                    }
                }
                if (head && half == 0) __stcg(lbase + h, l > 0.f ? (m_used + log2f(l)) * kLn2 : -INFINITY);
                umma::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar + B_O_FREE);
                if (split) {
                    // the last unit of the group to finish merges the group's split partials
                    __threadfence();
                    named_barrier_sync(kSmBar, 128);
                    if (tid == 0) s_misc[2] = (atomicAdd(a.done + grp, 1) == u.n_chunks - 1) ? 1 : 0;
                    named_barrier_sync(kSmBar, 128);
                    const int is_last = *reinterpret_cast<volatile int*>(s_misc + 2);
                    named_barrier_sync(kSmBar, 128);
                    if (is_last) {
                        __threadfence();
                        merge_slots(a, u.slot_base, u.n_chunks, 0, HQ, shard_out(a, u), shard_lse(a, u), tid >> 5, 4, tid & 31);
                        if (a.finish_ns) {
                            named_barrier_sync(kSmBar, 128);
                            if (tid == 0) record_finish(a, u.b);
                        }
                    }
                } else if (a.finish_ns) {
                    named_barrier_sync(kSmBar, 128);
                    if (tid == 0) record_finish(a, u.b);
                }
            }
            seq++;
        }
    }

    umma::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, 512);
    }
}

template <int HQ>
cudaError_t run(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s) {
    CUtensorMap tm;
    if (!make_tmap_2d(&tm, a.k_pages, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 576, (uint64_t)a.num_pages * a.page_size,
                      576 * 2, 64, kT, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    auto fn = mla_bf16_kernel<HQ>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    fn<<<g.ctas, kThreads, kSmemBytes, s>>>(tm, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_mla_bf16(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s) {
    switch (a.hq) {
        case 16: return run<16>(g, a, s);
        case 32: return run<32>(g, a, s);
        case 64: return run<64>(g, a, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace dcp
