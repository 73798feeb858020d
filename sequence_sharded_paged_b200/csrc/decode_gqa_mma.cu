// decode_gqa_mma.cu -- split-KV GQA decode attention on tensor cores, for a
// head group of 16 query heads per KV head (one m16 tile).
//
// "Efficient Decode Context Parallelism with vLLM for Long Context Workloads",
// section 4.1 ("Compute" on the local KV slice, partial output + LSE) and
// section 5.4 (each KV head broadcast to its query heads).
//
// Roofline: a group of 16 heads does 2*16*(D + D) = 64*D flop per token per KV
// head for 4*D bytes of K+V, i.e. 16 flop/byte: ~105 TFLOP/s at the measured
// 6.5 TB/s, beyond the CUDA-core fp32 rate but far below the tensor pipe, so
// the kernel is HBM-bound and uses warp-level mma.sync m16n8k16 (fp32
// accumulate): the 16 heads of a KV head fill M exactly, tokens are N.  Q K^T
// runs in bf16 (exact products); P V runs in bf16 on the V fragments as loaded,
// with P split into two bf16 terms (P_hi + P_lo, 16 significant bits).  The
// running maximum is rescaled lazily: only when a row's maximum grows by more
// than 2^8, so the 16 x D accumulator is rarely touched.
//
// Structure: persistent grid, one work unit (shard, request, chunk) per CTA
// iteration, all KV heads in the CTA.  Warp NCW (producer) issues TMA tiled
// loads of 16-token stages into a ring of shared-memory stages (mbarrier
// complete_tx): one 4-D box for K and one for V, which view the pool as
// [page * Hkv + head][64-column half][token][64 columns] and land as
// [head][half][16 tokens][128 B] with 128-byte swizzle (the copy engine's
// cost is per copy, so a stage is two copies rather than one per head and
// half).  Consumer warp w owns KV head
// w % Hkv and every (NCW/Hkv)-th stage: S = Q K^T (ldmatrix), online softmax
// in registers (quad shuffles), O += P V (ldmatrix.trans).  At the end of the
// unit the warps' states are merged through shared memory.
#include "common.cuh"
#include "finish.cuh"
#include "kernels.h"
#include "tma.h"

namespace dcp {

namespace {

constexpr int kTok = 16;            // tokens per stage
constexpr float kRescaleLog2 = 8.f;  // lazy rescale threshold (log2 units)
constexpr int kBoxBytes = kTok * 128;  // one [16][64] bf16 box (128-byte rows)

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// two floats -> bf16x2 high terms and bf16x2 residuals (x0 ~ hi.x + lo.x, x1 ~ hi.y + lo.y)
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// byte offset of (row r, column c) inside one [16][64] bf16 box with 128-byte swizzle
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)(r * 128 + ((((c >> 3) ^ (r & 7)) & 7) << 4) + ((c & 7) << 1));
}

// tmK / tmV: 4-D maps (one copy per stage each) when map4 != 0, else 2-D maps of
// [16 tokens][64 columns] boxes (one copy per head and half).
template <int D, int NCW>
__global__ void __launch_bounds__(32 * (NCW + 1), 1) gqa_mma_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                 const __grid_constant__ CUtensorMap tmV,
                                                                 DecodeArgs a, int stages, int map4) {
    constexpr int HALVES = D / 64;
    constexpr int NT = 32 * NCW;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int hkv = a.hkv;
    const uint32_t stage_bytes = (uint32_t)hkv * 2 * HALVES * kBoxBytes;  // K and V
    uint8_t* ring = smem;
    float* sO = reinterpret_cast<float*>(ring + (size_t)stages * stage_bytes);  // [hq][D]
    float* sM = sO + a.hq * D;                                                   // [NCW][16]
    float* sL = sM + NCW * 16;                                                   // [NCW][16]
    float* sLse = sL + NCW * 16;                                                 // [hq]
    float* sTot = sLse + a.hq;                                                   // [hq]
    uint64_t* full = reinterpret_cast<uint64_t*>(sTot + a.hq + (a.hq & 1));
    uint64_t* empty = full + stages;
    StageMeta* smeta = reinterpret_cast<StageMeta*>(empty + stages);
    __shared__ int s_flag;
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; s++) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, NCW);
        }
        s_abort = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int P = a.page_size;
    const int num_units = a.plan->num_units;

    if (warp == NCW) {
        if (lane != 0) return;
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        const uint64_t pol = l2_policy_evict_first();
        int stage = 0, issued = 0;
        uint32_t phase = 0;
        while (!s_abort) {
            const int ui = atomicAdd(a.ticket, 1);
            if (ui >= num_units) {
                if (mbar_wait(empty + stage, phase ^ 1, &s_abort, a.status)) {
                    smeta[stage] = StageMeta{-1, 0, 0, 0};
                    mbar_arrive(full + stage);
                }
                break;
            }
            const Unit u = a.units[ui];
            const int nst = (u.t1 - u.t0 + kTok - 1) / kTok;
            int k = 0;
            bool ok = true;
            do {
                if (!mbar_wait(empty + stage, phase ^ 1, &s_abort, a.status)) {
                    ok = false;
                    break;
                }
                const int t = u.t0 + k * kTok;
                int flags = (k == 0 ? kStageFirst : 0) | (k >= nst - 1 ? kStageLast : 0);
                if (nst == 0) {
                    smeta[stage] = StageMeta{ui, t, flags, k};
                    mbar_arrive(full + stage);
                } else {
                    const int j = t / P, sub = (t % P) / kTok;
                    const int pg = page_of(a, u.n, u.b, j);
                    if (pg >= 0) {
                        smeta[stage] = StageMeta{ui, t, flags | kStageValid, k};
                        mbar_arrive_expect_tx(full + stage, stage_bytes);
                        uint8_t* st = ring + (size_t)stage * stage_bytes;
                        if (map4) {
                            tma_load_4d(st, &tmK, 0, sub * kTok, 0, pg * hkv, full + stage, pol);
                            tma_load_4d(st + (size_t)hkv * HALVES * kBoxBytes, &tmV, 0, sub * kTok, 0, pg * hkv,
                                        full + stage, pol);
                        } else {
                            for (int g = 0; g < hkv; g++) {
                                const int row = (pg * hkv + g) * P + sub * kTok;
#pragma unroll
                                for (int h = 0; h < HALVES; h++) {
                                    tma_load_2d(st + ((size_t)(g * HALVES + h)) * kBoxBytes, &tmK, h * 64, row,
                                                full + stage, pol);
                                    tma_load_2d(st + ((size_t)((hkv + g) * HALVES + h)) * kBoxBytes, &tmV, h * 64,
                                                row, full + stage, pol);
                                }
                            }
                        }
                    } else {
                        record_status(a.status, DCP_ERR_UNALLOCATED_PAGE);
                        smeta[stage] = StageMeta{ui, t, flags, k};
                        mbar_arrive(full + stage);
                    }
                }
                issued++;
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1;
                }
                k++;
            } while (k < nst);
            if (!ok) break;
        }
        if (s_abort) {
            int n = issued < stages ? issued : stages;
            for (int k = 0; k < n; k++) {
                stage = stage == 0 ? stages - 1 : stage - 1;
                if (stage == stages - 1) phase ^= 1;
                mbar_wait(full + stage, phase, nullptr, a.status);
            }
        }
        return;
    }

    // consumer warp: KV head g, stage residue r of R
    const int R = NCW / hkv;
    const int g = warp % hkv;
    const int r = warp / hkv;
    const int qr = lane >> 2, qc = lane & 3;  // quad row / column
    // The 16 MMA rows of KV head g: with q_len query tokens per request, row r is
    // query token r / G of head g * G + r % G (G = heads per KV head); its output
    // row is (r / G) * (query heads) + g * G + r % G.
    const int G = 16 / a.q_len;
    const int hq_heads = a.hq / a.q_len;
    auto orow = [&](int gg, int rr) { return (rr / G) * hq_heads + gg * G + (rr % G); };
    const uint32_t ring_u32 = smem_u32(ring);
    int stage = 0;
    uint32_t phase = 0;
    uint32_t qa[D / 16][4];
    float o[D / 8][4];
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    int lim0 = 0x7fffffff, lim1 = 0x7fffffff;  // causal limits of rows qr and qr + 8
    Unit u = a.units[0];
    while (true) {
        if (!mbar_wait(full + stage, phase, &s_abort, a.status)) break;
        const StageMeta meta = load_meta(smeta + stage);
        if (meta.unit < 0) break;
        if (meta.flags & kStageFirst) {
            u = a.units[meta.unit];
            // Q fragments (A operand), 16 rows x D
            const uint32_t* q0 = reinterpret_cast<const uint32_t*>(a.q + ((int64_t)u.b * a.hq + orow(g, qr)) * D);
            const uint32_t* q1 = reinterpret_cast<const uint32_t*>(a.q + ((int64_t)u.b * a.hq + orow(g, qr + 8)) * D);
#pragma unroll
            for (int kk = 0; kk < D / 16; kk++) {
                qa[kk][0] = __ldg(q0 + (kk * 16 + 2 * qc) / 2);
                qa[kk][1] = __ldg(q1 + (kk * 16 + 2 * qc) / 2);
                qa[kk][2] = __ldg(q0 + (kk * 16 + 8 + 2 * qc) / 2);
                qa[kk][3] = __ldg(q1 + (kk * 16 + 8 + 2 * qc) / 2);
            }
            lim0 = row_limit(a, u, qr / G);
            lim1 = row_limit(a, u, (qr + 8) / G);
#pragma unroll
            for (int i = 0; i < D / 8; i++) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
            m0 = m1 = -INFINITY;
            l0 = l1 = 0.f;
        }
        {
            const int t = meta.t;
            const bool mine = (meta.sidx % R) == r;
            if (mine && (meta.flags & kStageValid)) {
                const int nvalid = min(u.t1 - t, kTok);
                const uint32_t kbase = ring_u32 + (uint32_t)stage * stage_bytes + (uint32_t)(g * HALVES) * kBoxBytes;
                const uint32_t vbase =
                    ring_u32 + (uint32_t)stage * stage_bytes + (uint32_t)((hkv + g) * HALVES) * kBoxBytes;
                // S = Q K^T : 16 heads x 16 tokens (two n-tiles)
                float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
                for (int kk = 0; kk < D / 16; kk++) {
                    const int tok = 8 * (mi >> 1) + rr;
                    const int col = (kk * 16 + 8 * (mi & 1));
                    const uint32_t addr = kbase + (uint32_t)(col / 64) * kBoxBytes + swz(tok, col & 63);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(addr, b0, b1, b2, b3);
                    mma_bf16(s[0], qa[kk], b0, b1);
                    mma_bf16(s[1], qa[kk], b2, b3);
                }
                // online softmax (log2 domain); rows qr and qr + 8, each cut by its causal limit
                const int nv0 = min(nvalid, max(0, lim0 - t)), nv1 = min(nvalid, max(0, lim1 - t));
                float x[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const int tok = nt * 8 + 2 * qc + (e & 1);
                        x[nt][e] = tok < (e < 2 ? nv0 : nv1) ? s[nt][e] * a.scale_log2 : -INFINITY;
                    }
                float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
                float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                // lazy rescale: the reference maximum moves only when a row's maximum grows by
                // more than 2^8 (p stays <= 2^8), so O is rarely rescaled
                float c0 = 1.f, c1 = 1.f;
                if (mx0 > m0 + kRescaleLog2 || (m0 == -INFINITY && mx0 != -INFINITY)) {
                    c0 = m0 == -INFINITY ? 0.f : fast_exp2(m0 - mx0);
                    m0 = mx0;
                }
                if (mx1 > m1 + kRescaleLog2 || (m1 == -INFINITY && mx1 != -INFINITY)) {
                    c1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - mx1);
                    m1 = mx1;
                }
                const float mn0 = m0 == -INFINITY ? 0.f : m0, mn1 = m1 == -INFINITY ? 0.f : m1;
                float p[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; nt++) {
                    p[nt][0] = fast_exp2(x[nt][0] - mn0);
                    p[nt][1] = fast_exp2(x[nt][1] - mn0);
                    p[nt][2] = fast_exp2(x[nt][2] - mn1);
                    p[nt][3] = fast_exp2(x[nt][3] - mn1);
                }
                l0 = l0 * c0 + p[0][0] + p[0][1] + p[1][0] + p[1][1];
                l1 = l1 * c1 + p[0][2] + p[0][3] + p[1][2] + p[1][3];
                if (c0 != 1.f || c1 != 1.f) {
#pragma unroll
                    for (int i = 0; i < D / 8; i++) {
                        o[i][0] *= c0;
                        o[i][1] *= c0;
                        o[i][2] *= c1;
                        o[i][3] *= c1;
                    }
                }
                // P V in bf16 with P = P_hi + P_lo (16 significant bits), V fragments as loaded
                uint32_t pa[4], pl[4];
                split_bf16(p[0][0], p[0][1], pa[0], pl[0]);
                split_bf16(p[0][2], p[0][3], pa[1], pl[1]);
                split_bf16(p[1][0], p[1][1], pa[2], pl[2]);
                split_bf16(p[1][2], p[1][3], pa[3], pl[3]);
                // rows past the unit's last token hold stale page contents: zero them so that
                // P = 0 cannot meet a NaN/Inf in the P V product
                if (nvalid < kTok) {
                    uint8_t* vrow = ring + (size_t)stage * stage_bytes + (size_t)((hkv + g) * HALVES) * kBoxBytes;
                    for (int i = lane; i < (kTok - nvalid) * 8 * HALVES; i += 32) {
                        const int h = i / ((kTok - nvalid) * 8), rem = i % ((kTok - nvalid) * 8);
                        *reinterpret_cast<uint4*>(vrow + h * kBoxBytes + (nvalid + rem / 8) * 128 + (rem % 8) * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    // order these generic-proxy writes before the next TMA write of this stage
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                }
                // O += P V : V^T fragments by ldmatrix.trans, two dv n-tiles per x4
#pragma unroll
                for (int jn = 0; jn < D / 8; jn += 2) {
                    const int tok = rr + 8 * (mi & 1);
                    const int col = 8 * (jn + (mi >> 1));
                    const uint32_t addr = vbase + (uint32_t)(col / 64) * kBoxBytes + swz(tok, col & 63);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(addr, b0, b1, b2, b3);
                    mma_bf16(o[jn], pa, b0, b1);
                    mma_bf16(o[jn + 1], pa, b2, b3);
                    mma_bf16(o[jn], pl, b0, b1);
                    mma_bf16(o[jn + 1], pl, b2, b3);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + stage);
        if (++stage == stages) {
            stage = 0;
            phase ^= 1;
        }
        if (!(meta.flags & kStageLast)) continue;
        // row sums over the quad
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        // merge the R warps of each KV head through shared memory: M, then rescaled sums
        if (qc == 0) {
            sM[warp * 16 + qr] = m0;
            sM[warp * 16 + qr + 8] = m1;
        }
        named_barrier_sync(1, NT);
        float M0 = -INFINITY, M1 = -INFINITY;
        for (int k = 0; k < R; k++) {
            M0 = fmaxf(M0, sM[(k * hkv + g) * 16 + qr]);
            M1 = fmaxf(M1, sM[(k * hkv + g) * 16 + qr + 8]);
        }
        const float w0 = (m0 == -INFINITY) ? 0.f : fast_exp2(m0 - M0);
        const float w1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - M1);
        if (qc == 0) {
            sL[warp * 16 + qr] = l0 * w0;
            sL[warp * 16 + qr + 8] = l1 * w1;
        }
        // accumulate O over the R warps of head g: warp r == 0 writes, then the others add in turn
        for (int k = 0; k < R; k++) {
            if (r == k) {
#pragma unroll
                for (int i = 0; i < D / 8; i++) {
                    float* row0 = sO + orow(g, qr) * D + i * 8 + 2 * qc;
                    float* row1 = sO + orow(g, qr + 8) * D + i * 8 + 2 * qc;
                    if (k == 0) {
                        row0[0] = o[i][0] * w0;
                        row0[1] = o[i][1] * w0;
                        row1[0] = o[i][2] * w1;
                        row1[1] = o[i][3] * w1;
                    } else {
                        row0[0] += o[i][0] * w0;
                        row0[1] += o[i][1] * w0;
                        row1[0] += o[i][2] * w1;
                        row1[1] += o[i][3] * w1;
                    }
                }
            }
            named_barrier_sync(1, NT);
        }
        // normalise and LSE (natural log)
        const int tid = threadIdx.x;
        for (int i = tid; i < a.hq; i += NT) {
            // output row i = (query token j, head hh): KV head hh / G, MMA row j * G + hh % G
            const int j = i / hq_heads, hh = i - j * hq_heads;
            const int gg = hh / G, row = j * G + hh % G;
            float M = -INFINITY, Ls = 0.f;
            for (int k = 0; k < R; k++) M = fmaxf(M, sM[(k * hkv + gg) * 16 + row]);
            for (int k = 0; k < R; k++) Ls += sL[(k * hkv + gg) * 16 + row];
            sLse[i] = (M == -INFINITY || Ls == 0.f) ? -INFINITY : (M + log2f(Ls)) * kLn2;
            sTot[i] = Ls;
        }
        named_barrier_sync(1, NT);
        for (int i = tid; i < a.hq * D; i += NT) {
            const int h = i / D;
            const float Ls = sTot[h];
            sO[i] = Ls > 0.f ? sO[i] / Ls : 0.f;
        }
        named_barrier_sync(1, NT);
        finish_unit<NT>(a, u, 0, 1, 0, a.hq, sO, sLse, &s_flag, tid, 1);
        named_barrier_sync(1, NT);
    }
}

template <int D, int NCW>
size_t gqa_mma_smem(int hq, int hkv, int stages) {
    const size_t stage_bytes = (size_t)hkv * 2 * (D / 64) * kBoxBytes;
    return 1024 + (size_t)stages * stage_bytes + (size_t)(hq * D + 2 * NCW * 16 + 2 * hq + 2) * 4 +
           (size_t)2 * stages * 8 + (size_t)stages * sizeof(StageMeta);
}

template <int D, int NCW>
int gqa_mma_stages(int hq, int hkv) {
    const size_t stage_bytes = (size_t)hkv * 2 * (D / 64) * kBoxBytes;
    const size_t fixed = gqa_mma_smem<D, NCW>(hq, hkv, 0);
    size_t n = (200 * 1024 - fixed) / (stage_bytes + 16 + sizeof(StageMeta));
    return (int)(n < 2 ? 2 : (n > 8 ? 8 : n));
}

template <int D, int NCW>
cudaError_t run(const DecodeGeometry& geo, const DecodeArgs& a, cudaStream_t s) {
    CUtensorMap tk, tv;
    // [page * Hkv + head][half][token][64 columns] view of each pool; the box is a whole
    // stage: 64 columns x 16 tokens x every half x every head
    const uint64_t dims[4] = {64, (uint64_t)a.page_size, (uint64_t)(D / 64), (uint64_t)a.num_pages * a.hkv};
    const uint64_t strides[3] = {(uint64_t)D * 2, 128, (uint64_t)a.page_size * D * 2};
    const uint32_t box[4] = {64, (uint32_t)kTok, (uint32_t)(D / 64), (uint32_t)a.hkv};
    int map4 = make_tmap_4d(&tk, a.k_pages, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dims, strides, box,
                            CU_TENSOR_MAP_SWIZZLE_128B) &&
               make_tmap_4d(&tv, a.v_pages, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dims, strides, box,
                            CU_TENSOR_MAP_SWIZZLE_128B);
    if (!map4) {
        const uint64_t rows = (uint64_t)a.num_pages * a.hkv * a.page_size;
        if (!make_tmap_2d(&tk, a.k_pages, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, D, rows, (uint64_t)D * 2, 64, kTok,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_tmap_2d(&tv, a.v_pages, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, D, rows, (uint64_t)D * 2, 64, kTok,
                          CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    const int stages = gqa_mma_stages<D, NCW>(a.hq, a.hkv);
    const size_t smem = gqa_mma_smem<D, NCW>(a.hq, a.hkv, stages);
    cudaError_t e = cudaFuncSetAttribute(gqa_mma_kernel<D, NCW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    gqa_mma_kernel<D, NCW><<<geo.ctas, 32 * (NCW + 1), smem, s>>>(tk, tv, a, stages, map4);
    return cudaGetLastError();
}

}  // namespace

bool gqa_mma_supported(int hq, int hkv, int dk) {
    return hq == 16 * hkv && (hkv == 1 || hkv == 2 || hkv == 4 || hkv == 8) && (dk == 64 || dk == 128);
}

int gqa_mma_blocks_per_sm(int hq, int hkv, int dk) {
    const int ncw = hkv > 4 ? 8 : 4;
    const void* fn;
    size_t smem;
    if (dk == 64) {
        fn = ncw == 8 ? (const void*)gqa_mma_kernel<64, 8> : (const void*)gqa_mma_kernel<64, 4>;
        smem = ncw == 8 ? gqa_mma_smem<64, 8>(hq, hkv, gqa_mma_stages<64, 8>(hq, hkv))
                        : gqa_mma_smem<64, 4>(hq, hkv, gqa_mma_stages<64, 4>(hq, hkv));
    } else {
        fn = ncw == 8 ? (const void*)gqa_mma_kernel<128, 8> : (const void*)gqa_mma_kernel<128, 4>;
        smem = ncw == 8 ? gqa_mma_smem<128, 8>(hq, hkv, gqa_mma_stages<128, 8>(hq, hkv))
                        : gqa_mma_smem<128, 4>(hq, hkv, gqa_mma_stages<128, 4>(hq, hkv));
    }
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, 32 * (ncw + 1), smem) != cudaSuccess) return 0;
    return n;
}

cudaError_t launch_decode_gqa_mma(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s) {
    const bool wide = a.hkv > 4;
    if (a.dk == 64) return wide ? run<64, 8>(g, a, s) : run<64, 4>(g, a, s);
    if (a.dk == 128) return wide ? run<128, 8>(g, a, s) : run<128, 4>(g, a, s);
    return cudaErrorNotSupported;
}

}  // namespace dcp
