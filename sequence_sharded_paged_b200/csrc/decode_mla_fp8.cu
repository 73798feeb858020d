// decode_mla_fp8.cu -- split-KV MLA decode attention over an fp8 (e4m3) latent
// cache with a per-token fp32 scale, on 5th-generation tensor cores with 8-bit
// operands (tcgen05 kind::f8f6f4): the cache is never widened.
//
// Method: "Efficient Decode Context Parallelism with vLLM for Long Context
// Workloads", section 4.1 ("Compute": the gathered query against the local KV
// slice, partial output + LSE) and section 5.3 (MLA, absorbed: key = the whole
// 576-wide latent row, value = its first 512 entries).
//
// Value of a latent element = e4m3 code * s_t (s_t = per-token scale).
//
// Scores.  Each head's bf16 query row is scaled by a power of two sigma_h
// (largest |q| sigma_h in [128, 256)) and split exactly into two e4m3 terms,
// q sigma_h = q_hi + q_lo (bf16 has 8 significant bits, e4m3 4; only elements
// below ~2^-17 of the row maximum lose bits).  The two terms are stacked as
// the 128 rows of one operand:
//   [S_hi; S_lo] = [Q_hi; Q_lo] . C^T   M = 128, N = 64 tokens, K = 576 (e4m3 x e4m3)
// so 18 MMAs per 64-token tile read the raw page.  Lanes 0..63 of TMEM hold
// S_hi, lanes 64..127 S_lo; the softmax warps exchange halves through shared
// memory and form s = scale * s_t * (S_hi + S_lo) / sigma_h.
//
// Values.  O^T = V^T . P'^T with V^T read MN-major straight from the raw tile
// (e4m3) and P' = 16 * p * s_t split into three e5m2 terms (about nine
// significant bits: relative error below 2^-9 of P, inside the fp8 tolerance;
// e5m2's exponent range covers p * s_t without per-token rescaling):
//   O^T += V^T . P'_j^T   M = 128 value columns (4 blocks), N = Hq, K = 64, j = 0..2
// 24 MMAs per tile.  O = O^T / (16 * l).  The running maximum is rescaled
// lazily (O^T only when a head's maximum grows by more than 2^8).
//
// Tiles: one 64-token page per tile, nine [64 rows][64 B] TMA boxes with
// 64-byte swizzle (36 KB) + 256 B of scales; three stages in flight.
//
// Warp roles (one CTA per SM, persistent, units from an atomic ticket):
//   warp 0      TMA producer (lane 0)
//   warp 1      TMEM allocation, MMA issue (lane 0, event loop)
//   warps 2..5  q split, softmax, lazy rescale of O^T, epilogue; the warp on TMEM
//               quadrant q owns heads 32 (q & 1) .. +31 and tokens 32 (q >> 1) .. +31
#include "common.cuh"
#include "finish.cuh"
#include "kernels.h"
#include "tma.h"
#include "umma.cuh"

namespace dcp {

namespace {

constexpr int kT = 64;                     // tokens per tile (one page)
constexpr int kKB = 9;                     // 576 = 9 blocks of 64 bytes
constexpr int kBox = kT * 64;              // [64 rows][64 B] box: 4 KB
constexpr int kTileBytes = kKB * kBox;     // 36864
constexpr int kQBox = 128 * 64;            // [128 rows][64 B]: 8 KB
constexpr int kQBytes = kKB * kQBox;       // 73728
constexpr int kStages = 3;
constexpr int kPTerm = 64 * 64;            // P'_j^T [64 heads][64 tokens] e5m2: 4 KB
constexpr int kPBuf = 3 * kPTerm;          // 12 KB
constexpr float kRescaleLog2 = 8.f;
constexpr float kPScale = 16.f;            // P' = 16 p s_t
constexpr int kSmBar = 1;
constexpr int kThreads = 192;

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffTiles = kQBytes;
constexpr uint32_t kOffScales = kOffTiles + kStages * kTileBytes;
constexpr uint32_t kOffP = (kOffScales + kStages * kT * 4 + 1023) / 1024 * 1024;
constexpr uint32_t kOffX = kOffP + 2 * kPBuf;                 // [2 halves][64 heads][32] f32
constexpr uint32_t kOffXmax = kOffX + 2 * 64 * 32 * 4;        // [2][64] f32
constexpr uint32_t kOffBars = kOffXmax + 2 * 64 * 4;
constexpr uint32_t kOffMeta = kOffBars + 32 * 8;
constexpr uint32_t kOffSmall = kOffMeta + kStages * 16;
constexpr uint32_t kSmemBytes = kOffSmall + (6 * 64 + 16) * 4 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

enum : int {
    B_TILE_FULL = 0,   // [3]
    B_TILE_EMPTY = 3,  // [3]
    B_S_FULL = 6,      // [2]
    B_P_FULL = 8,      // [2]
    B_PV_DONE = 10,    // [2]
    B_Q_FULL = 12,
    B_Q_FREE = 13,
    B_O_FREE = 14,
    B_FINAL = 15,
};

// byte offset of 16-byte chunk c (0..3) of row r in a 64-byte-swizzled block
__device__ __forceinline__ uint32_t sw64(int r, int c) { return (uint32_t)(r * 64 + (((c ^ (r >> 1)) & 3) << 4)); }

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

// two floats -> two 8-bit codes (round to nearest even, saturating to the largest finite value)
__device__ __forceinline__ uint32_t to_e4m3x2(float a, float b) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ uint32_t to_e5m2x2(float a, float b) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E5M2);
}
__device__ __forceinline__ float2 from_fp8x2(uint32_t c, __nv_fp8_interpretation_t k) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(c & 0xFFFF), k);
    return __half22float2(*reinterpret_cast<__half2*>(&h));
}

template <int HQ>
__global__ void __launch_bounds__(kThreads, 1)
    mla_fp8_kernel(const __grid_constant__ CUtensorMap tmC, DecodeArgs a) {
    constexpr uint32_t IDESC_S = umma::idesc_f8(umma::kE4M3, umma::kE4M3, 0, 0, 128, kT);
    constexpr uint32_t IDESC_PV = umma::idesc_f8(umma::kE4M3, umma::kE5M2, 1, 0, 128, HQ);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kOffBars);
    StageMeta* tmeta = reinterpret_cast<StageMeta*>(sm + kOffMeta);
    float* xbuf = reinterpret_cast<float*>(sm + kOffX);
    float* xmax = reinterpret_cast<float*>(sm + kOffXmax);
    float* s_m = reinterpret_cast<float*>(sm + kOffSmall);
    float* s_l0 = s_m + 64;
    float* s_l1 = s_l0 + 64;
    float* s_alpha = s_l1 + 64;
    float* s_qs = s_alpha + 64;   // 1 / sigma_h
    int* s_misc = reinterpret_cast<int*>(s_qs + 128);  // [0] tmem base, [2] split flag, [3] abort
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_misc + 3);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sm_u32 = smem_u32(sm);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; i++) {
            mbar_init(bar + B_TILE_FULL + i, 1);
            mbar_init(bar + B_TILE_EMPTY + i, 1);
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
        *s_abort = 0;
        fence_barrier_init();
    }
    // Q rows of heads >= HQ stay zero for the whole kernel
    for (int i = threadIdx.x; i < kQBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(sm + kOffQ)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (warp == 1) umma::tmem_alloc(reinterpret_cast<uint32_t*>(s_misc), 512);
    umma::fence_proxy_async_smem();
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(s_misc);
    const uint32_t t_o = tmem;         // O^T: columns [blk*HQ, blk*HQ + HQ)
    const uint32_t t_s = tmem + 256;   // S buffers: [256 + 64 sb, +64)
    const int num_units = a.plan->num_units;
    const int P = a.page_size;

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            tma_prefetch_desc(&tmC);
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
                    if (!mbar_wait(bar + B_TILE_EMPTY + stage, phase ^ 1, s_abort, a.status)) {
                        ok = false;
                        break;
                    }
                    if (done) {
                        tmeta[stage] = StageMeta{-1, 0, 0, 0};
                        mbar_arrive(bar + B_TILE_FULL + stage);
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
                    tmeta[stage] = StageMeta{ui, t, flags | ((pg >= 0 ? nvalid : 0) << 8), k};
                    if (pg >= 0) {
                        mbar_arrive_expect_tx(bar + B_TILE_FULL + stage, kTileBytes + kT * 4);
                        uint8_t* dst = sm + kOffTiles + (size_t)stage * kTileBytes;
                        const int32_t row0 = pg * P + (t % P);
#pragma unroll
                        for (int kb = 0; kb < kKB; kb++)
                            tma_load_2d(dst + kb * kBox, &tmC, kb * 64, row0, bar + B_TILE_FULL + stage, pol);
                        bulk_g2s(sm + kOffScales + stage * kT * 4, a.kv_scales + row0, kT * 4,
                                 bar + B_TILE_FULL + stage);
                    } else {
                        mbar_arrive(bar + B_TILE_FULL + stage);
                    }
                    issued++;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                    k++;
                } while (k < nt);
            }
            if (*s_abort) {  // bounded drain of copies still in flight
                int n = issued < kStages ? issued : kStages;
                for (int i = 0; i < n; i++) {
                    stage = stage == 0 ? kStages - 1 : stage - 1;
                    if (stage == kStages - 1) phase ^= 1;
                    mbar_wait(bar + B_TILE_FULL + stage, phase, nullptr, a.status);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer (event loop)
        if (lane == 0) {
            const uint64_t dq0 = umma::smem_desc(sm_u32 + kOffQ, 16, 512, umma::kSw64);
            const uint64_t dt0 = umma::smem_desc(sm_u32 + kOffTiles, 16, 512, umma::kSw64);
            const uint64_t dv0 = umma::smem_desc(sm_u32 + kOffTiles, kBox, 512, umma::kSw64);
            const uint64_t dp0 = umma::smem_desc(sm_u32 + kOffP, 16, 512, umma::kSw64);
            uint32_t next_s = 0, next_pv = 0, unit_k = 0, ofree_k = 0;
            uint32_t first_bits = 0;  // bit b: the tile in S buffer b opened its unit
            bool sentinel = false;
            uint64_t t_prog = global_timer_ns();
            while (true) {
                bool progress = false;
                if (next_pv < next_s) {
                    const int pb = next_pv & 1;
                    const bool fst = (first_bits >> pb) & 1;
                    if (mbar_test(bar + B_P_FULL + pb, (next_pv >> 1) & 1) &&
                        (!fst || mbar_test(bar + B_O_FREE, (ofree_k & 1) ^ 1))) {
                        if (fst) ofree_k++;
                        umma::fence_after_sync();
                        const int st = next_pv % kStages;
                        const uint64_t tile = (uint64_t)((st * kTileBytes) >> 4);
                        const uint64_t pbuf = (uint64_t)((pb * kPBuf) >> 4);
#pragma unroll
                        for (int j = 0; j < 3; j++)
#pragma unroll
                            for (int blk = 0; blk < 4; blk++)
#pragma unroll
                                for (int ks = 0; ks < 2; ks++) {
                                    const uint64_t ad = dv0 + tile + (uint64_t)(((2 * blk) * kBox + ks * 2048) >> 4);
                                    const uint64_t bd = dp0 + pbuf + (uint64_t)((j * kPTerm + ks * 32) >> 4);
                                    umma::mma_f8(t_o + blk * HQ, ad, bd, IDESC_PV, (fst && j == 0 && ks == 0) ? 0u : 1u);
                                }
                        umma::commit(bar + B_PV_DONE + pb);
                        umma::commit(bar + B_TILE_EMPTY + st);
                        next_pv++;
                        progress = true;
                    }
                }
                if (!sentinel && next_s - next_pv < 2) {
                    const int st = next_s % kStages;
                    if (mbar_test(bar + B_TILE_FULL + st, (next_s / kStages) & 1)) {
                        const StageMeta meta = load_meta(tmeta + st);
                        if (meta.unit < 0) {
                            sentinel = true;
                        } else {
                            const bool first = meta.flags & kStageFirst;
                            if (!first || mbar_test(bar + B_Q_FULL, unit_k & 1)) {
                                if (first) unit_k++;
                                umma::fence_after_sync();
                                const int sb = next_s & 1;
                                const uint64_t tile = (uint64_t)((st * kTileBytes) >> 4);
#pragma unroll
                                for (int kb = 0; kb < kKB; kb++)
#pragma unroll
                                    for (int ks = 0; ks < 2; ks++) {
                                        const uint64_t aq = dq0 + (uint64_t)((kb * kQBox + ks * 32) >> 4);
                                        const uint64_t bt = dt0 + tile + (uint64_t)((kb * kBox + ks * 32) >> 4);
                                        umma::mma_f8(t_s + sb * kT, aq, bt, IDESC_S, (kb | ks) ? 1u : 0u);
                                    }
                                umma::commit(bar + B_S_FULL + sb);
                                if (meta.flags & kStageLast) umma::commit(bar + B_Q_FREE);
                                first_bits = (first_bits & ~(1u << sb)) | ((first ? 1u : 0u) << sb);
                                next_s++;
                                progress = true;
                            }
                        }
                    }
                }
                if (sentinel && next_pv == next_s) break;
                if (progress) {
                    t_prog = global_timer_ns();
                } else {
                    if (*s_abort) break;
                    if (global_timer_ns() - t_prog > kWaitLimitNs) {
                        record_status(a.status, DCP_ERR_TIMEOUT);
                        *s_abort = 1;
                        break;
                    }
                }
            }
            umma::commit(bar + B_FINAL);
            mbar_wait(bar + B_FINAL, 0, nullptr, a.status);
        }
    } else {
        // ------------------------------------------------------------------ q split, softmax, epilogue
        const int qd = warp & 3;                    // TMEM lane quadrant
        const int h = 32 * (qd & 1) + lane;         // head
        const int half = qd >> 1;                   // 0: holds S_hi, finishes tokens 0..31; 1: S_lo, tokens 32..63
        const bool head = h < HQ;
        const int tid = threadIdx.x - 64;           // 0..127
        const int sw = warp - 2;                    // 0..3
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        uint32_t seq = 0, unit_k = 0;
        float m_used = -INFINITY, lpart = 0.f;
        bool o_has = false, fail = false;
        Unit u;
        u.n = u.b = u.t0 = u.t1 = u.slot = u.n_chunks = u.slot_base = u.pad = 0;
        float* xrow_out = xbuf + ((size_t)half * 64 + h) * 32;        // my half of the exchange
        const float* xrow_in = xbuf + ((size_t)(half ^ 1) * 64 + h) * 32;
        while (true) {
            const int st = seq % kStages;
            const int sb = seq & 1;
            if (!fail) fail = !mbar_wait(bar + B_TILE_FULL + st, (seq / kStages) & 1, s_abort, a.status);
            StageMeta meta{-1, 0, 0, 0};
            if (!fail) meta = load_meta(tmeta + st);
            if (named_barrier_or(kSmBar, 128, fail)) break;
            if (meta.unit < 0) break;
            const bool first = meta.flags & kStageFirst;
            const bool last = meta.flags & kStageLast;
            const int nvalid = (meta.flags >> 8) & 0xFF;
            if (first) {
                u = a.units[meta.unit];
                // the previous unit's S MMAs are complete (first unit passes at once)
                fail = !mbar_wait(bar + B_Q_FREE, (unit_k & 1) ^ 1, s_abort, a.status);
                if (!fail) {
                    // warp sw splits heads sw*16 .. sw*16+15 of request u.b; lane c handles
                    // 16-element chunk c (and c + 32 for c < 4) of the 576-wide row
                    for (int hh = sw * 16; hh < sw * 16 + 16 && hh < HQ; hh++) {
                        const uint4* qrow = reinterpret_cast<const uint4*>(a.q + ((int64_t)u.b * HQ + hh) * 576);
                        uint4 w[2][2];
                        float amax = 0.f;
#pragma unroll
                        for (int k2 = 0; k2 < 2; k2++) {
                            const int c = lane + 32 * k2;
                            if (c < 36) {
                                w[k2][0] = __ldg(qrow + 2 * c);
                                w[k2][1] = __ldg(qrow + 2 * c + 1);
                                const uint32_t ws[8] = {w[k2][0].x, w[k2][0].y, w[k2][0].z, w[k2][0].w,
                                                        w[k2][1].x, w[k2][1].y, w[k2][1].z, w[k2][1].w};
#pragma unroll
                                for (int e = 0; e < 8; e++)
                                    amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(ws[e])), fabsf(bf16_hi(ws[e]))));
                            }
                        }
#pragma unroll
                        for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                        int ex = 0;
                        frexpf(amax, &ex);                       // amax in [2^(ex-1), 2^ex)
                        ex = max(ex, -110);                       // sigma and 1/sigma stay finite
                        const float sig = amax > 0.f ? ldexpf(1.f, 8 - ex) : 1.f;
                        if (lane == 0) s_qs[hh] = 1.f / sig;
#pragma unroll
                        for (int k2 = 0; k2 < 2; k2++) {
                            const int c = lane + 32 * k2;
                            if (c < 36) {
                                const uint32_t ws[8] = {w[k2][0].x, w[k2][0].y, w[k2][0].z, w[k2][0].w,
                                                        w[k2][1].x, w[k2][1].y, w[k2][1].z, w[k2][1].w};
                                uint32_t hi[4], lo[4];
#pragma unroll
                                for (int e = 0; e < 4; e++) {
                                    const float a0 = bf16_lo(ws[2 * e]) * sig, a1 = bf16_hi(ws[2 * e]) * sig;
                                    const float a2 = bf16_lo(ws[2 * e + 1]) * sig, a3 = bf16_hi(ws[2 * e + 1]) * sig;
                                    const uint32_t h01 = to_e4m3x2(a0, a1), h23 = to_e4m3x2(a2, a3);
                                    const float2 d01 = from_fp8x2(h01, __NV_E4M3), d23 = from_fp8x2(h23, __NV_E4M3);
                                    const uint32_t l01 = to_e4m3x2(a0 - d01.x, a1 - d01.y);
                                    const uint32_t l23 = to_e4m3x2(a2 - d23.x, a3 - d23.y);
                                    hi[e] = h01 | (h23 << 16);
                                    lo[e] = l01 | (l23 << 16);
                                }
                                // chunk c: bytes [16c, 16c+16) of the row = box c/4, 16-byte chunk c%4
                                uint8_t* qb = sm + kOffQ + (c >> 2) * kQBox;
                                *reinterpret_cast<uint4*>(qb + sw64(hh, c & 3)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                                *reinterpret_cast<uint4*>(qb + sw64(64 + hh, c & 3)) =
                                    make_uint4(lo[0], lo[1], lo[2], lo[3]);
                            }
                        }
                    }
                    umma::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar + B_Q_FULL);
                }
                unit_k++;
                m_used = -INFINITY;
                lpart = 0.f;
                o_has = false;
            }
            // ---- scores: S_hi / S_lo rows, exchange halves
            if (!fail) fail = !mbar_wait(bar + B_S_FULL + sb, (seq >> 1) & 1, s_abort, a.status);
            umma::fence_after_sync();
            uint32_t mine[32], other[32];
            umma::ld32(t_s + lane_off + sb * kT, mine);
            umma::ld32(t_s + lane_off + sb * kT + 32, other);
            umma::wait_ld();
            // half 0 keeps tokens 0..31 and sends 32..63; half 1 the reverse
#pragma unroll
            for (int j = 0; j < 32; j++) {
                const uint32_t m0 = half ? other[j] : mine[j], o0 = half ? mine[j] : other[j];
                mine[j] = m0;
                other[j] = o0;
            }
#pragma unroll
            for (int c = 0; c < 8; c++)   // rotated 16-byte chunks: no bank conflicts
                *reinterpret_cast<uint4*>(xrow_out + (((c + h) & 7) << 2)) =
                    make_uint4(other[4 * c], other[4 * c + 1], other[4 * c + 2], other[4 * c + 3]);
            named_barrier_sync(kSmBar, 128);
            const int base = half ? 32 : 0;  // my tokens
            float x[32];
            {
                const float* tsc = reinterpret_cast<const float*>(sm + kOffScales + st * kT * 4) + base;
                const float f = head ? s_qs[h] * a.scale_log2 : 0.f;
#pragma unroll
                for (int c = 0; c < 8; c++) {
                    const float4 o4 = *reinterpret_cast<const float4*>(xrow_in + (((c + h) & 7) << 2));
                    const float ov[4] = {o4.x, o4.y, o4.z, o4.w};
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const int j = 4 * c + e;
                        const float s = __uint_as_float(mine[j]) + ov[e];
                        x[j] = (base + j < nvalid) ? s * f * tsc[j] : -INFINITY;
                    }
                }
            }
            float mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; j++) mt = fmaxf(mt, x[j]);
            xmax[half * 64 + h] = mt;
            named_barrier_sync(kSmBar, 128);
            mt = fmaxf(mt, xmax[(half ^ 1) * 64 + h]);
            float alpha = 1.f;
            if (mt > m_used + kRescaleLog2 || (m_used == -INFINITY && mt != -INFINITY)) {
                alpha = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - mt);
                m_used = mt;
            }
            if (half == 0) s_alpha[h] = alpha;
            // one barrier: some head rescaled while O^T holds data, or a wait failed (a failing
            // thread republishes the abort flag first, so every thread reads it set after the barrier)
            if (fail) *s_abort = 1;
            const int any = named_barrier_or(kSmBar, 128, fail || (head && alpha != 1.f && o_has));
            if (any && *s_abort) break;
            if (any) {
                // the previous tile's P V must be complete before O^T is rescaled
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
            // ---- P' = 16 p s_t as three e5m2 terms (the P buffer is free once P V of tile seq-2 is done)
            if (!fail) fail = !mbar_wait(bar + B_PV_DONE + sb, ((seq >> 1) & 1) ^ 1, s_abort, a.status);
            if (!fail && head) {
                const float* tsc = reinterpret_cast<const float*>(sm + kOffScales + st * kT * 4) + base;
                float rowsum = 0.f;
                uint32_t t0[8], t1[8], t2[8];
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    float pp[4];
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const float p = x[j + e] == -INFINITY ? 0.f : fast_exp2(x[j + e] - m_used);
                        rowsum += p;
                        pp[e] = p > 0.f ? p * tsc[j + e] * kPScale : 0.f;  // stale scales meet no p = 0
                    }
                    uint32_t c0[2], c1[2], c2[2];
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const float a0 = pp[2 * e], a1 = pp[2 * e + 1];
                        c0[e] = to_e5m2x2(a0, a1);
                        const float2 d0 = from_fp8x2(c0[e], __NV_E5M2);
                        const float r0 = a0 - d0.x, r1 = a1 - d0.y;
                        c1[e] = to_e5m2x2(r0, r1);
                        const float2 d1 = from_fp8x2(c1[e], __NV_E5M2);
                        c2[e] = to_e5m2x2(r0 - d1.x, r1 - d1.y);
                    }
                    t0[j / 4] = c0[0] | (c0[1] << 16);
                    t1[j / 4] = c1[0] | (c1[1] << 16);
                    t2[j / 4] = c2[0] | (c2[1] << 16);
                }
                lpart = lpart * alpha + rowsum;
                uint8_t* pb = sm + kOffP + sb * kPBuf;
                // my 32 tokens = 16-byte chunks 2*half and 2*half + 1 of row h
#pragma unroll
                for (int cc = 0; cc < 2; cc++) {
                    const int c = 2 * half + cc;
                    *reinterpret_cast<uint4*>(pb + 0 * kPTerm + sw64(h, c)) =
                        make_uint4(t0[4 * cc], t0[4 * cc + 1], t0[4 * cc + 2], t0[4 * cc + 3]);
                    *reinterpret_cast<uint4*>(pb + 1 * kPTerm + sw64(h, c)) =
                        make_uint4(t1[4 * cc], t1[4 * cc + 1], t1[4 * cc + 2], t1[4 * cc + 3]);
                    *reinterpret_cast<uint4*>(pb + 2 * kPTerm + sw64(h, c)) =
                        make_uint4(t2[4 * cc], t2[4 * cc + 1], t2[4 * cc + 2], t2[4 * cc + 3]);
                }
            } else if (!fail) {
                lpart = lpart * alpha;
            }
            if (!fail && nvalid < kT) {
                // rows past the last valid token hold stale page bytes (possibly NaN codes):
                // zero their value columns so that P = 0 cannot meet them
                uint8_t* tile = sm + kOffTiles + (size_t)st * kTileBytes;
                const int nr = kT - nvalid;
                for (int i = tid; i < nr * 4 * 8; i += 128) {
                    const int box = i / (nr * 4), rem = i - box * nr * 4;
                    const int r = nvalid + rem / 4, c = rem & 3;
                    *reinterpret_cast<uint4*>(tile + box * kBox + r * 64 + c * 16) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            umma::fence_proxy_async_smem();
            umma::fence_before_sync();
            __syncwarp();
            if (!fail && lane == 0) mbar_arrive(bar + B_P_FULL + sb);
            o_has = true;
            // ---- end of unit: O = O^T / (16 l), LSE
            if (last) {
                if (!fail) fail = !mbar_wait(bar + B_PV_DONE + sb, (seq >> 1) & 1, s_abort, a.status);
                umma::fence_after_sync();
                (half ? s_l1 : s_l0)[h] = lpart;
                if (half == 0) s_m[h] = m_used;
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
                            const float l = s_l0[c0 + i] + s_l1[c0 + i];
                            __stcg(obase + (int64_t)(c0 + i) * 512 + dv,
                                   l > 0.f ? __uint_as_float(r[i]) / (kPScale * l) : 0.f);
                        }
                    }
                }
                if (half == 0 && head) {
                    const float l = s_l0[h] + s_l1[h];
                    __stcg(lbase + h, l > 0.f ? (s_m[h] + log2f(l)) * kLn2 : -INFINITY);
                }
                umma::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar + B_O_FREE);
                if (split) {
                    __threadfence();
                    named_barrier_sync(kSmBar, 128);
                    if (tid == 0) s_misc[2] = (atomicAdd(a.done + shard, 1) == u.n_chunks - 1) ? 1 : 0;
                    named_barrier_sync(kSmBar, 128);
                    const int is_last = *reinterpret_cast<volatile int*>(s_misc + 2);
                    named_barrier_sync(kSmBar, 128);
                    if (is_last) {
                        __threadfence();
                        merge_split_chunks(a, u, shard, 0, HQ, tid, 128);
                    }
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
    if (!make_tmap_2d(&tm, a.k_pages, CU_TENSOR_MAP_DATA_TYPE_UINT8, 576, (uint64_t)a.num_pages * a.page_size, 576, 64,
                      kT, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    auto fn = mla_fp8_kernel<HQ>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    fn<<<g.ctas, kThreads, kSmemBytes, s>>>(tm, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_mla_fp8(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s) {
    switch (a.hq) {
        case 16: return run<16>(g, a, s);
        case 32: return run<32>(g, a, s);
        case 64: return run<64>(g, a, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace dcp
