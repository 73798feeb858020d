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
// Query.  A small kernel splits each head's bf16 query row exactly into two
// e4m3 terms after scaling it by a power of two sigma_h (largest |q| sigma_h in
// [128, 256)): q sigma_h = q_hi + q_lo (bf16 has 8 significant bits, e4m3 4;
// only elements below ~2^-17 of the row maximum lose bits).  Rows are stacked
// 128 high: for heads 16 j .. 16 j + 15, rows 32 j .. 32 j + 15 hold q_hi and
// rows 32 j + 16 .. 32 j + 31 hold q_lo, so that a head's two score rows land
// in one warp's TMEM lane quadrant.  The first 512 columns of those rows live
// in tensor memory (the MMA's A operand), the 64 rope columns in shared memory.
//
// Scores.  [S_hi; S_lo] = [Q_hi; Q_lo] . C^T, M = 128, K = 576, over a tile of
// one or two pages (N = 64 or 128 tokens): 16 MMAs with A in TMEM + 2 with A in
// shared memory; the pages are the only shared-memory operand.  Lane pairs
// (l, l + 16) swap halves with shuffles and form
// s = scale * s_t * (S_hi + S_lo) / sigma_h.
//
// Values.  O^T = V^T . W^T with V^T read MN-major straight from the raw pages
// and W = p * s_t in two e4m3 terms (relative error below 2^-8).  The running
// maximum m absorbs the tile's largest scale (m >= max_t (x_t + log2 s_t), x in
// log2 units), so W = 2^(x - m) s_t <= 2^8 stays inside e4m3's range whatever
// the scales; it is rescaled lazily (O^T only when m grows by more than 2^8).
//   O^T += V^T . W_j^T   M = 128 value columns (4 blocks), N = Hq, K = 64 per page, j = 0, 1
// 16 MMAs per page.  O = O^T / l with l = sum_t 2^(x_t - m).
//
// Pages: nine [64 rows][64 B] TMA boxes with 64-byte swizzle (36 KB) + 256 B of
// scales, in a ring of five slots laid out [block][slot][64 rows][64 B], so that
// two adjacent slots form one 128-row operand.  A tile pairs a page with the next
// one unless the page sits in the last slot or closes its unit.  A slot is
// refilled as soon as P V of its page completes.
//
// Warp roles (one CTA per SM, persistent, units from an atomic ticket):
//   warp 0      producer: tickets, page indices (one page of lookahead), TMA
//   warp 1      TMEM allocation; issues the scores of each tile
//   warps 2..9  query rows, softmax, lazy rescale of O^T, epilogue.  The two
//               warps on TMEM quadrant j own heads 16 j .. 16 j + 15: warp
//               group g (warps 2..5: g = 0, 6..9: g = 1) page g of the tile,
//               in which lane l < 16 takes tokens 0..31 and lane l + 16 tokens
//               32..63; g also picks the value blocks 2 g, 2 g + 1 that the warp
//               rescales and stores.
//   warp 10     issues P V of each tile
#include "common.cuh"
#include "finish.cuh"
#include "kernels.h"
#include "tma.h"
#include "umma.cuh"

namespace dcp {

// Optional timeline of CTA 0 (SM clock at each protocol step), compiled only
// with -DDCP_TRACE for profiling builds; expands to nothing otherwise.
#ifdef DCP_TRACE
__device__ unsigned long long g_mla8_trace[40][512];
#define TRACE(ev, k)                                                          \
    do {                                                                      \
        if (blockIdx.x == 0 && (k) < 512) g_mla8_trace[ev][(k)] = clock64();  \
    } while (0)
extern "C" int dcp_trace8_read(unsigned long long* host) {
    return (int)cudaMemcpyFromSymbol(host, g_mla8_trace, sizeof(g_mla8_trace));
}
#else
#define TRACE(ev, k) \
    do {             \
    } while (0)
#endif

namespace {

constexpr int kPg = 64;                    // tokens per page = tokens per tile
constexpr int kKB = 9;                     // 576 = 9 blocks of 64 bytes
constexpr int kBox = kPg * 64;             // [64 rows][64 B] box: 4 KB
constexpr int kTileBytes = kKB * kBox;     // one page: 36864
constexpr int kSlots = 5;                  // pages in flight
constexpr int kKbStride = kSlots * kBox;   // block kb of every slot is contiguous: [kb][slot][64 rows][64 B]
constexpr int kRopeBytes = 128 * 64;       // rope columns of the 128 query rows
constexpr int kPTerm = 64 * 64;            // W_j^T of one page [64 heads][64 tokens] e4m3: 4 KB
constexpr int kPPage = 2 * kPTerm;         // both terms of one page
constexpr int kPBuf = 2 * kPPage;          // a tile of two pages: 16 KB
constexpr float kRescaleLog2 = 8.f;
constexpr int kSmBar = 1;                  // the 256 softmax threads
constexpr int kSoftWarps = 8;
constexpr int kThreads = 32 * (3 + kSoftWarps);  // producer, S issuer, softmax x 8, P V issuer
constexpr uint32_t kColO = 0, kColS = 256, kColQ = 384;  // TMEM columns

constexpr uint32_t kOffTiles = 0;
constexpr uint32_t kOffRope = kOffTiles + kSlots * kTileBytes;
constexpr uint32_t kOffP = kOffRope + kRopeBytes;
constexpr uint32_t kOffScales = kOffP + 2 * kPBuf;
constexpr uint32_t kOffBars = kOffScales + kSlots * kPg * 4;
constexpr uint32_t kOffMeta = kOffBars + 32 * 8;
constexpr uint32_t kOffSmall = kOffMeta + kSlots * 16;
// s_alpha[64], s_inv[64], s_gmax[2][64], s_gl[2][64], misc[16]
constexpr uint32_t kSmemBytes = kOffSmall + (6 * 64 + 16) * 4 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffRope % 1024 == 0 && kOffP % 1024 == 0, "swizzled operands need 1 KB alignment");

enum : int {
    B_PAGE_FULL = 0,    // [kSlots]
    B_PAGE_EMPTY = 8,   // [kSlots]
    B_S_FULL = 16,
    B_S_FREE = 17,
    B_P_FULL = 20,      // [2]
    B_PV_DONE = 22,     // [2]
    B_Q_FULL = 24,
    B_Q_FREE = 25,
    B_O_FREE = 26,
    B_FINAL = 27,
};

// Page (= tile) k of the ring sequence uses slot k mod 5 and completes phase (k / 5) & 1
// of that slot's barriers.
__device__ __forceinline__ int slot_of(uint32_t k) { return (int)(k % kSlots); }
__device__ __forceinline__ uint32_t phase_of(uint32_t k) { return (k / kSlots) & 1; }

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

// two floats -> two e4m3 codes (round to nearest even, saturating)
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float a, float b) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t c) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(c & 0xFFFF), __NV_E4M3);
    return __half22float2(*reinterpret_cast<__half2*>(&h));
}
// w0, w1 >= 0 -> two-term e4m3 codes (hi, lo) with w ~ hi + lo, via f16 (11 bits)
__device__ __forceinline__ void split_e4m3x2(float w0, float w1, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(w0, w1);
    const __nv_fp8x2_storage_t c =
        __nv_cvt_halfraw2_to_fp8x2(*reinterpret_cast<const __half2_raw*>(&h), __NV_SATFINITE, __NV_E4M3);
    __half2_raw br = __nv_cvt_fp8x2_to_halfraw2(c, __NV_E4M3);
    const __half2 r = __hsub2(h, *reinterpret_cast<__half2*>(&br));  // exact
    hi = (uint32_t)c;
    lo = (uint32_t)__nv_cvt_halfraw2_to_fp8x2(*reinterpret_cast<const __half2_raw*>(&r), __NV_SATFINITE, __NV_E4M3);
}
// 32 weights -> two e4m3 terms, four codes per word
__device__ __forceinline__ void split32(const float (&w)[32], uint32_t (&chi)[8], uint32_t (&clo)[8]) {
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
        uint32_t h01, l01, h23, l23;
        split_e4m3x2(w[j], w[j + 1], h01, l01);
        split_e4m3x2(w[j + 2], w[j + 3], h23, l23);
        chi[j / 4] = h01 | (h23 << 16);
        clo[j / 4] = l01 | (l23 << 16);
    }
}

// A tile is one page, or two when the page is not in the last slot (so the next page's
// slot is adjacent) and does not close its unit.  Producer order makes the next page the
// next one of the same unit then.
__device__ __forceinline__ bool pairs_with_next(int slot, const StageMeta& m) {
    return slot != kSlots - 1 && !(m.flags & kStageLast);
}

// ------------------------------------------------------------------------------------------
// Query split: one warp per (request, head).  Writes rows hi / lo of qs[b][128][576] and
// qinv[b][64] = 1 / sigma_h.
__global__ void __launch_bounds__(128) mla_fp8_qsplit_kernel(const __nv_bfloat16* __restrict__ q, int B, int HQ,
                                                             uint8_t* __restrict__ qs, float* __restrict__ qinv) {
    const int gw = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (gw >= B * HQ) return;
    const int b = gw / HQ, h = gw - b * HQ;
    const uint4* qrow = reinterpret_cast<const uint4*>(q + ((int64_t)b * HQ + h) * 576);
    // lane handles 16-element chunks c = lane and c = lane + 32 (< 36)
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
            for (int e = 0; e < 8; e++) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(ws[e])), fabsf(bf16_hi(ws[e]))));
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int ex = 0;
    frexpf(amax, &ex);      // amax in [2^(ex-1), 2^ex)
    ex = max(ex, -110);     // sigma and 1/sigma stay finite
    const float sig = amax > 0.f ? ldexpf(1.f, 8 - ex) : 1.f;
    if (lane == 0) qinv[(int64_t)b * 64 + h] = 1.f / sig;
    uint8_t* hi_row = qs + ((int64_t)b * 128 + 32 * (h >> 4) + (h & 15)) * 576;
    uint8_t* lo_row = hi_row + 16 * 576;
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
                const uint32_t h01 = f32x2_to_e4m3x2(a0, a1), h23 = f32x2_to_e4m3x2(a2, a3);
                const float2 d01 = e4m3x2_to_f32x2(h01), d23 = e4m3x2_to_f32x2(h23);
                hi[e] = h01 | (h23 << 16);
                lo[e] = f32x2_to_e4m3x2(a0 - d01.x, a1 - d01.y) | (f32x2_to_e4m3x2(a2 - d23.x, a3 - d23.y) << 16);
            }
            *reinterpret_cast<uint4*>(hi_row + 16 * c) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(lo_row + 16 * c) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
    }
}

// ------------------------------------------------------------------------------------------
template <int HQ>
__global__ void __launch_bounds__(kThreads, 1)
    mla_fp8_kernel(const __grid_constant__ CUtensorMap tmC, DecodeArgs a) {
    constexpr uint32_t IDESC_S = umma::idesc_f8(umma::kE4M3, umma::kE4M3, 0, 0, 128, kPg);
    constexpr uint32_t IDESC_S128 = umma::idesc_f8(umma::kE4M3, umma::kE4M3, 0, 0, 128, 2 * kPg);
    constexpr uint32_t IDESC_PV = umma::idesc_f8(umma::kE4M3, umma::kE4M3, 1, 0, 128, HQ);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kOffBars);
    StageMeta* tmeta = reinterpret_cast<StageMeta*>(sm + kOffMeta);  // per page slot
    float* s_alpha = reinterpret_cast<float*>(sm + kOffSmall);
    float* s_inv = s_alpha + 64;
    float* s_gmax = s_inv + 64;     // [2 pages][64 heads]: each page's bound on x + log2 s
    float* s_gl = s_gmax + 128;     // [2][64]
    int* s_misc = reinterpret_cast<int*>(s_gl + 128);  // [0] tmem base, [2] split flag, [3] abort
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_misc + 3);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sm_u32 = smem_u32(sm);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kSlots; i++) {
            mbar_init(bar + B_PAGE_FULL + i, 1);
            mbar_init(bar + B_PAGE_EMPTY + i, 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(bar + B_P_FULL + i, kSoftWarps);
            mbar_init(bar + B_PV_DONE + i, 1);
        }
        mbar_init(bar + B_S_FULL, 1);
        mbar_init(bar + B_S_FREE, kSoftWarps);
        mbar_init(bar + B_Q_FULL, kSoftWarps);
        mbar_init(bar + B_Q_FREE, 1);
        mbar_init(bar + B_O_FREE, kSoftWarps);
        mbar_init(bar + B_FINAL, 2);
        *s_abort = 0;
        fence_barrier_init();
    }
    // rope rows of heads >= HQ stay zero for the whole kernel
    for (int i = threadIdx.x; i < kRopeBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(sm + kOffRope)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (warp == 1) umma::tmem_alloc(reinterpret_cast<uint32_t*>(s_misc), 512);
    umma::fence_proxy_async_smem();
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(s_misc);
    const uint32_t t_o = tmem + kColO;  // O^T: columns [blk*HQ, blk*HQ + HQ)
    const uint32_t t_s = tmem + kColS;  // S buffers: [kColS + 64 sb, +64)
    const uint32_t t_q = tmem + kColQ;  // query rows, first 512 columns (128 TMEM columns)
    const int num_units = a.plan->num_units;
    const int P = a.page_size;

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        // One page of lookahead: the next page's unit and index are fetched before the slot
        // wait, so their latency overlaps it.  Lane 0 takes tickets and handles the barriers;
        // lanes 0..8 then issue the page's nine boxes and lane 9 its scales at once.
        const uint64_t pol = l2_policy_evict_first();
        if (lane == 0) tma_prefetch_desc(&tmC);
        int ui = -1, k = 0, nt = 0;
        Unit u{};
        // moves (ui, k) to the next page (the same on every lane); false when no work is left
        auto advance = [&]() -> bool {
            if (ui >= 0 && k + 1 < nt) {
                k++;
                return true;
            }
            int nu = 0;
            if (lane == 0) nu = atomicAdd(a.ticket, 1);
            ui = __shfl_sync(0xffffffffu, nu, 0);
            if (ui >= num_units) return false;
            u = a.units[ui];
            nt = max(1, (u.t1 - u.t0 + kPg - 1) / kPg);  // an empty unit still yields one tile
            k = 0;
            return true;
        };
        auto page = [&]() -> int {
            const int t = u.t0 + k * kPg;
            return (u.t1 - t > 0) ? page_of(a, u.n, u.b, t / P) : -1;
        };
        bool have = advance();
        int pg = have ? page() : -1;
        uint32_t ps = 0;  // pages issued into the ring
        while (true) {
            const bool c_have = have;
            const int c_ui = ui, c_k = k, c_nt = nt, c_pg = pg;
            const Unit c_u = u;
            if (have) {
                have = advance();
                if (have) pg = page();
            }
            const int slot = slot_of(ps);
            int waited = 1;
            if (lane == 0) waited = mbar_wait(bar + B_PAGE_EMPTY + slot, phase_of(ps) ^ 1, s_abort, a.status);
            if (!__shfl_sync(0xffffffffu, waited, 0)) break;
            if (lane == 0) TRACE(14, ps);
            if (!c_have) {
                if (lane == 0) {
                    tmeta[slot] = StageMeta{-1, 0, 0, 0};
                    mbar_arrive(bar + B_PAGE_FULL + slot);
                }
                break;
            }
            const int t = c_u.t0 + c_k * kPg;
            int nvalid = max(0, min(c_u.t1 - t, kPg));
            if (nvalid > 0 && c_pg < 0) {
                if (lane == 0) record_status(a.status, DCP_ERR_UNALLOCATED_PAGE);
                nvalid = 0;
            }
            const int flags = (c_k == 0 ? kStageFirst : 0) | (c_k == c_nt - 1 ? kStageLast : 0);
            if (lane == 0) tmeta[slot] = StageMeta{c_ui, t, flags | (nvalid << 8), c_k};
            if (nvalid > 0) {
                if (lane == 0) mbar_arrive_expect_tx(bar + B_PAGE_FULL + slot, kTileBytes + kPg * 4);
                __syncwarp();
                const int32_t row0 = c_pg * P;
                if (lane < kKB)
                    tma_load_2d(sm + kOffTiles + lane * kKbStride + slot * kBox, &tmC, lane * 64, row0,
                                bar + B_PAGE_FULL + slot, pol);
                else if (lane == kKB)
                    bulk_g2s(sm + kOffScales + slot * kPg * 4, a.kv_scales + row0, kPg * 4, bar + B_PAGE_FULL + slot);
            } else if (lane == 0) {
                mbar_arrive(bar + B_PAGE_FULL + slot);
            }
            if (lane == 0) TRACE(15, ps);
            ps++;
        }
        if (lane == 0 && *s_abort) {  // bounded drain of copies still in flight
            const uint32_t n = ps < (uint32_t)kSlots ? ps : (uint32_t)kSlots;
            for (uint32_t i = 1; i <= n; i++)
                mbar_wait(bar + B_PAGE_FULL + slot_of(ps - i), phase_of(ps - i), nullptr, a.status);
        }
    } else if (warp == 1 || warp == 2 + kSoftWarps) {
        // ------------------------------------------------------------------ MMA issuers
        // Two threads: warp 1 issues the scores of each page as soon as its page, its S buffer
        // and its unit's query rows are ready; the last warp issues P V of each page when the
        // softmax has written its weights.  Each thread's waits hide behind the other's MMAs.
        if (lane == 0) {
            uint32_t unit_k = 0, ofree_k = 0;
            if (warp == 1) {
                const uint64_t dr0 = umma::smem_desc(sm_u32 + kOffRope, 16, 512, umma::kSw64);
                const uint64_t dt0 = umma::smem_desc(sm_u32 + kOffTiles, 16, 512, umma::kSw64);
                for (uint32_t kk = 0, tt = 0;; tt++) {
                    const int slot = slot_of(kk);
                    if (!mbar_wait(bar + B_PAGE_FULL + slot, phase_of(kk), s_abort, a.status)) break;
                    const StageMeta m0 = load_meta(tmeta + slot);
                    if (m0.unit < 0) break;
                    const bool pair = pairs_with_next(slot, m0);
                    StageMeta m1 = m0;
                    if (pair) {
                        if (!mbar_wait(bar + B_PAGE_FULL + slot + 1, phase_of(kk + 1), s_abort, a.status)) break;
                        m1 = load_meta(tmeta + slot + 1);
                    }
                    // the softmax has read the previous tile's scores
                    if (tt >= 1 && !mbar_wait(bar + B_S_FREE, (tt - 1) & 1, s_abort, a.status)) break;
                    if (m0.flags & kStageFirst) {
                        if (!mbar_wait(bar + B_Q_FULL, unit_k & 1, s_abort, a.status)) break;
                        unit_k++;
                    }
                    TRACE(0, tt);
                    umma::fence_after_sync();
                    const uint32_t idesc = pair ? IDESC_S128 : IDESC_S;
                    const uint64_t dt = dt0 + (uint64_t)((slot * kBox) >> 4);
#pragma unroll
                    for (int kb = 0; kb < 8; kb++)
#pragma unroll
                        for (int ks = 0; ks < 2; ks++)
                            umma::mma_f8_ts(t_s, t_q + (2 * kb + ks) * 8, dt + (uint64_t)((kb * kKbStride + ks * 32) >> 4),
                                            idesc, (kb | ks) ? 1u : 0u);
#pragma unroll
                    for (int ks = 0; ks < 2; ks++)
                        umma::mma_f8(t_s, dr0 + (uint64_t)((ks * 32) >> 4),
                                     dt + (uint64_t)((8 * kKbStride + ks * 32) >> 4), idesc, 1u);
                    umma::commit(bar + B_S_FULL);
                    if (m1.flags & kStageLast) umma::commit(bar + B_Q_FREE);
                    TRACE(1, tt);
                    kk += pair ? 2 : 1;
                }
            } else {
                const uint64_t dv0 = umma::smem_desc(sm_u32 + kOffTiles, kKbStride, 512, umma::kSw64);
                const uint64_t dp0 = umma::smem_desc(sm_u32 + kOffP, 16, 512, umma::kSw64);
                for (uint32_t kk = 0, tt = 0;; tt++) {
                    const int slot = slot_of(kk);
                    // the page's metadata stays in place until this thread releases the slot
                    if (!mbar_wait(bar + B_PAGE_FULL + slot, phase_of(kk), s_abort, a.status)) break;
                    const StageMeta m0 = load_meta(tmeta + slot);
                    if (m0.unit < 0) break;
                    const bool pair = pairs_with_next(slot, m0);
                    const int pb = tt & 1;
                    if (!mbar_wait(bar + B_P_FULL + pb, (tt >> 1) & 1, s_abort, a.status)) break;
                    const bool fst = m0.flags & kStageFirst;
                    if (fst) {
                        if (!mbar_wait(bar + B_O_FREE, (ofree_k & 1) ^ 1, s_abort, a.status)) break;
                        ofree_k++;
                    }
                    TRACE(2, tt);
                    umma::fence_after_sync();
                    for (int g = 0; g < (pair ? 2 : 1); g++) {
                        const int sl = slot + g;
                        const uint64_t da = dv0 + (uint64_t)((sl * kBox) >> 4);
                        const uint64_t db = dp0 + (uint64_t)((pb * kPBuf + g * kPPage) >> 4);
                        // consecutive MMAs go to different accumulator blocks
#pragma unroll
                        for (int j = 0; j < 2; j++)
#pragma unroll
                            for (int ks = 0; ks < 2; ks++)
#pragma unroll
                                for (int blk = 0; blk < 4; blk++)
                                    umma::mma_f8(t_o + blk * HQ,
                                                 da + (uint64_t)((2 * blk * kKbStride + ks * 2048) >> 4),
                                                 db + (uint64_t)((j * kPTerm + ks * 32) >> 4), IDESC_PV,
                                                 (fst && g == 0 && j == 0 && ks == 0) ? 0u : 1u);
                        umma::commit(bar + B_PAGE_EMPTY + sl);
                    }
                    umma::commit(bar + B_PV_DONE + pb);
                    TRACE(4, tt);
                    kk += pair ? 2 : 1;
                }
            }
            umma::commit(bar + B_FINAL);
            mbar_wait(bar + B_FINAL, 0, nullptr, a.status);
        }
    } else {
        // ------------------------------------------------------------------ query rows, softmax, epilogue
        const int qd = warp & 3;                  // TMEM lane quadrant
        const int wg = (warp - 2) >> 2;           // token group = page wg of the tile
        const int half = lane >> 4;               // 0: row holds S_hi; 1: S_lo
        const int h = 16 * qd + (lane & 15);      // head
        const bool head = h < HQ;
        const int row = 32 * qd + lane;           // query row = TMEM lane
        const int base = 32 * half;               // my 32 tokens of the page
        const int tid = threadIdx.x - 64;         // 0..255
        const int gtid = tid & 127;               // index within the token group
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        uint32_t seq = 0, kk = 0, unit_k = 0;
        float m_used = -INFINITY, lpart = 0.f, f = 0.f;
        int lim = 0x7fffffff;  // local tokens [0, lim) of the unit's shard this row attends
        bool o_has = false, fail = false;
        Unit u{};
        while (true) {
            const int pb = seq & 1;
            const int slot0 = slot_of(kk);
            if (!fail) fail = !mbar_wait(bar + B_PAGE_FULL + slot0, phase_of(kk), s_abort, a.status);
            StageMeta m0{-1, 0, 0, 0};
            if (!fail) m0 = load_meta(tmeta + slot0);
            if (named_barrier_or(kSmBar, 256, fail)) break;
            if (m0.unit < 0) break;
            const bool pair = pairs_with_next(slot0, m0);
            StageMeta m1 = m0;
            if (pair) {
                if (!fail) fail = !mbar_wait(bar + B_PAGE_FULL + slot0 + 1, phase_of(kk + 1), s_abort, a.status);
                if (!fail) m1 = load_meta(tmeta + slot0 + 1);
            }
            const bool first = m0.flags & kStageFirst;
            const bool last = m1.flags & kStageLast;
            const bool mine = wg == 0 || pair;          // does my page exist in this tile
            const int my_slot = mine ? slot0 + wg : slot0;
            const int nvalid = mine ? (((wg ? m1.flags : m0.flags) >> 8) & 0xFF) : 0;
            const bool page_full = nvalid == kPg;
            if (first) {
                u = a.units[m0.unit];
                f = head ? __ldg(a.qinv + (int64_t)u.b * 64 + h) * a.scale_log2 : 0.f;
                lim = head ? row_limit(a, u, h / (HQ / a.q_len)) : 0x7fffffff;
                // the previous unit's S MMAs are complete (first unit passes at once)
                fail = fail || !mbar_wait(bar + B_Q_FREE, (unit_k & 1) ^ 1, s_abort, a.status);
                if (!fail) {
                    if (head) {
                        // token group wg copies query bytes [256 wg, 256 wg + 256) -> TMEM columns 64 wg ..
                        const uint4* src = reinterpret_cast<const uint4*>(a.qs + ((int64_t)u.b * 128 + row) * 576);
                        uint4 v[16];
#pragma unroll
                        for (int i = 0; i < 16; i++) v[i] = __ldg(src + 16 * wg + i);
                        uint32_t r0[32], r1[32];
#pragma unroll
                        for (int i = 0; i < 8; i++) {
                            r0[4 * i] = v[i].x;
                            r0[4 * i + 1] = v[i].y;
                            r0[4 * i + 2] = v[i].z;
                            r0[4 * i + 3] = v[i].w;
                            r1[4 * i] = v[8 + i].x;
                            r1[4 * i + 1] = v[8 + i].y;
                            r1[4 * i + 2] = v[8 + i].z;
                            r1[4 * i + 3] = v[8 + i].w;
                        }
                        umma::st32(t_q + lane_off + 64 * wg, r0);
                        umma::st32(t_q + lane_off + 64 * wg + 32, r1);
                        if (wg == 1) {
#pragma unroll
                            for (int c = 0; c < 4; c++)
                                *reinterpret_cast<uint4*>(sm + kOffRope + sw64(row, c)) = __ldg(src + 32 + c);
                        }
                    }
                    umma::wait_st();
                    umma::fence_proxy_async_smem();
                    umma::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar + B_Q_FULL);
                }
                unit_k++;
                m_used = -INFINITY;
                lpart = 0.f;
                o_has = false;
            }
            // tokens of my page this row attends: the page's valid tokens, cut by the row's
            // causal limit when the request has several query tokens
            const int row_nv = min(nvalid, max(0, lim - (wg ? m1.t : m0.t)));
            const bool full = row_nv == kPg;
            // ---- scores of my page: rows S_hi (lane < 16) and S_lo (lane >= 16) of head h; swap halves
            if (!fail) fail = !mbar_wait(bar + B_S_FULL, seq & 1, s_abort, a.status);
            umma::fence_after_sync();
            if (threadIdx.x == 64) TRACE(5, seq);
            if (lane == 0) TRACE(24 + warp - 2, seq);
            const float4* tsc4 = reinterpret_cast<const float4*>(sm + kOffScales + (my_slot * kPg + base) * 4);
            float x[32];
            float smax = 0.f;
            {
                uint32_t v0[32], v1[32];
                umma::ld32(t_s + lane_off + 64 * wg, v0);
                umma::ld32(t_s + lane_off + 64 * wg + 32, v1);
                umma::wait_ld();
                // the S columns may be overwritten by the next tile's MMAs from here on
                umma::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar + B_S_FREE);
#pragma unroll
                for (int j4 = 0; j4 < 8; j4++) {
                    const float4 sc4 = tsc4[j4];
                    const float sc[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const int j = 4 * j4 + e;
                        const uint32_t keep = half ? v1[j] : v0[j], send = half ? v0[j] : v1[j];
                        const float sv =
                            __uint_as_float(keep) + __uint_as_float(__shfl_xor_sync(0xffffffffu, send, 16));
                        x[j] = sv * f * sc[e];
                        smax = fmaxf(smax, sc[e]);
                    }
                }
                if (!full) {
                    // tokens past the end of the unit (or no page): no score, and their stale
                    // scales do not count
                    smax = 0.f;
#pragma unroll
                    for (int j4 = 0; j4 < 8; j4++) {
                        const float4 sc4 = tsc4[j4];
                        const float sc[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            const bool valid = base + 4 * j4 + e < row_nv;
                            x[4 * j4 + e] = valid ? x[4 * j4 + e] : -INFINITY;
                            smax = valid ? fmaxf(smax, sc[e]) : smax;
                        }
                    }
                }
            }
            if (threadIdx.x == 64) TRACE(6, seq);
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; j++) mx = fmaxf(mx, x[j]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 16));
            // Bound of this page: m_g = max_t x_t + log2 max_t s_t >= x_t + log2 s_t for its tokens;
            // the tile's bound is the larger of the two pages' (the weights 2^(x - m) s_t stay <= 2^8).
            // A head's running maximum moves iff one of its pages' bounds passes the threshold, so
            // one barrier both exchanges the bounds and decides whether any head rescales.
            const float mt_g = (mx == -INFINITY || !(smax > 0.f)) ? mx : mx + __log2f(smax);
            if (half == 0) s_gmax[wg * 64 + h] = mt_g;
            const bool moves = mt_g > m_used + kRescaleLog2 || (m_used == -INFINITY && mt_g != -INFINITY);
            if (threadIdx.x == 64) TRACE(7, seq);
            // (a failing thread republishes the abort flag first, so every thread reads it set after
            // the barrier)
            if (fail) *s_abort = 1;
            const int any = named_barrier_or(kSmBar, 256, fail || (head && moves && o_has));
            if (any && *s_abort) break;
            const float mt = fmaxf(mt_g, s_gmax[(wg ^ 1) * 64 + h]);
            float alpha = 1.f;
            if (mt > m_used + kRescaleLog2 || (m_used == -INFINITY && mt != -INFINITY)) {
                alpha = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - mt);
                m_used = mt;
            }
            if (threadIdx.x == 64) TRACE(8, seq);
            if (any) {
                if (half == 0 && wg == 0) s_alpha[h] = alpha;
                named_barrier_sync(kSmBar, 256);
                // the previous tile's P V must be complete before O^T is rescaled; token group wg
                // rescales value blocks 2 wg, 2 wg + 1 of its lane quadrant
                fail = !mbar_wait(bar + B_PV_DONE + (pb ^ 1), ((seq - 1) >> 1) & 1, s_abort, a.status);
                if (!fail) {
                    umma::fence_after_sync();
#pragma unroll 1
                    for (int blk = 2 * wg; blk < 2 * wg + 2; blk++) {
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
            // ---- W = p s_t as two e4m3 terms (the P buffer is free once P V of tile seq-2 is done)
            if (!fail) fail = !mbar_wait(bar + B_PV_DONE + pb, ((seq >> 1) & 1) ^ 1, s_abort, a.status);
            if (threadIdx.x == 64) TRACE(10, seq);
            if (!fail && head && mine) {
                float w[32];
                float rowsum = 0.f;
                if (m_used != -INFINITY) {
                    // 2^(-inf - m) = 0 for masked tokens; stale scales are zeroed below
#pragma unroll
                    for (int j4 = 0; j4 < 8; j4++) {
                        const float4 sc4 = tsc4[j4];
                        const float sc[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            const float p = fast_exp2(x[4 * j4 + e] - m_used);
                            rowsum += p;
                            w[4 * j4 + e] = p * sc[e];
                        }
                    }
                    if (!full) {
#pragma unroll
                        for (int j = 0; j < 32; j++) w[j] = (base + j < row_nv) ? w[j] : 0.f;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; j++) w[j] = 0.f;
                }
                uint32_t chi[8], clo[8];
                split32(w, chi, clo);
                lpart = lpart * alpha + rowsum;
                // page wg of the tile, row h, 16-byte chunks 2 half and 2 half + 1
                uint8_t* pbuf = sm + kOffP + pb * kPBuf + wg * kPPage;
#pragma unroll
                for (int cc = 0; cc < 2; cc++) {
                    const uint32_t off = sw64(h, 2 * half + cc);
                    *reinterpret_cast<uint4*>(pbuf + off) =
                        make_uint4(chi[4 * cc], chi[4 * cc + 1], chi[4 * cc + 2], chi[4 * cc + 3]);
                    *reinterpret_cast<uint4*>(pbuf + kPTerm + off) =
                        make_uint4(clo[4 * cc], clo[4 * cc + 1], clo[4 * cc + 2], clo[4 * cc + 3]);
                }
            } else if (!fail) {
                lpart = lpart * alpha;
            }
            if (!fail && mine && !page_full) {
                // rows past the last valid token hold stale page bytes (possibly NaN codes):
                // zero their value columns so that W = 0 cannot meet them (token group wg
                // clears its own page)
                uint8_t* tile = sm + kOffTiles + my_slot * kBox;
                const int nr = kPg - nvalid;
                for (int i = gtid; i < nr * 4 * 8; i += 128) {
                    const int kb = i / (nr * 4), rem = i - kb * nr * 4;
                    const int r = nvalid + rem / 4, c = rem & 3;
                    *reinterpret_cast<uint4*>(tile + kb * kKbStride + r * 64 + c * 16) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            umma::fence_proxy_async_smem();
            umma::fence_before_sync();
            __syncwarp();
            if (!fail && lane == 0) mbar_arrive(bar + B_P_FULL + pb);
            if (threadIdx.x == 64) TRACE(9, seq);
            if (lane == 0) TRACE(16 + warp - 2, seq);
            o_has = true;
            // ---- end of unit: O = O^T / l, LSE
            if (last) {
                if (threadIdx.x == 64) TRACE(12, seq);
                if (!fail) fail = !mbar_wait(bar + B_PV_DONE + pb, (seq >> 1) & 1, s_abort, a.status);
                umma::fence_after_sync();
                const float lg = lpart + __shfl_xor_sync(0xffffffffu, lpart, 16);  // this token group
                if (half == 0) s_gl[wg * 64 + h] = lg;
                const int64_t grp = u.grp;
                const bool split = u.n_chunks > 1;
                float* obase = split ? a.split_o + (int64_t)u.slot * a.hq * 512 : a.o_partial + grp * a.hq * 512;
                float* lbase = split ? a.split_lse + (int64_t)u.slot * a.hq : a.lse + grp * a.hq;
                if (named_barrier_or(kSmBar, 256, fail)) break;
                if (head && half == 0 && wg == 0) {
                    const float l = lg + s_gl[64 + h];
                    s_inv[h] = l > 0.f ? 1.f / l : 0.f;
                    __stcg(lbase + h, l > 0.f ? (m_used + log2f(l)) * kLn2 : -INFINITY);
                }
                named_barrier_sync(kSmBar, 256);
#pragma unroll 1
                for (int c0 = 0; c0 < HQ; c0 += 16) {
                    float inv[16];
#pragma unroll
                    for (int i = 0; i < 16; i++) inv[i] = s_inv[c0 + i];
#pragma unroll 1
                    for (int blk = 2 * wg; blk < 2 * wg + 2; blk++) {
                        const int dv = blk * 128 + 32 * qd + lane;
                        uint32_t r[16];
                        umma::ld16(t_o + lane_off + blk * HQ + c0, r);
                        umma::wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; i++)
                            __stcg(obase + (int64_t)(c0 + i) * 512 + dv, __uint_as_float(r[i]) * inv[i]);
                    }
                }
                umma::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar + B_O_FREE);
                if (split) {
                    __threadfence();
                    named_barrier_sync(kSmBar, 256);
                    if (tid == 0) s_misc[2] = (atomicAdd(a.done + grp, 1) == u.n_chunks - 1) ? 1 : 0;
                    named_barrier_sync(kSmBar, 256);
                    const int is_last = *reinterpret_cast<volatile int*>(s_misc + 2);
                    named_barrier_sync(kSmBar, 256);
                    if (is_last) {
                        __threadfence();
                        merge_slots(a, u.slot_base, u.n_chunks, 0, HQ, shard_out(a, u), shard_lse(a, u), tid >> 5, 8, tid & 31);
                        if (a.finish_ns) {
                            named_barrier_sync(kSmBar, 256);
                            if (tid == 0) record_finish(a, u.b);
                        }
                    }
                } else if (a.finish_ns) {
                    named_barrier_sync(kSmBar, 256);
                    if (tid == 0) record_finish(a, u.b);
                }
                if (threadIdx.x == 64) TRACE(13, seq);
            }
            if (threadIdx.x == 64) TRACE(11, seq);
            seq++;
            kk += pair ? 2 : 1;
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
                      kPg, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    const int warps = a.batch * HQ;
    mla_fp8_qsplit_kernel<<<(warps + 3) / 4, 128, 0, s>>>(a.q, a.batch, HQ, a.qs, a.qinv);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    auto fn = mla_fp8_kernel<HQ>;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    fn<<<g.ctas, kThreads, kSmemBytes, s>>>(tm, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_mla_fp8(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s) {
    if (!a.qs || !a.qinv) return cudaErrorInvalidValue;
    switch (a.hq) {
        case 16: return run<16>(g, a, s);
        case 32: return run<32>(g, a, s);
        case 64: return run<64>(g, a, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace dcp
