// decode_simt.cu -- split-KV decode attention on CUDA cores.
//
// "Compute" step of "Efficient Decode Context Parallelism with vLLM for Long
// Context Workloads", section 4.1: the query against one shard's local KV
// slice, giving a partial output and its LSE.  GQA (section 5.4): KV head g
// serves query heads g*G .. g*G+G-1.  MLA (section 5.3): every head reads the
// 576-wide latent row; the value is its first 512 entries.
//
// Structure (both kernels): a persistent grid; each CTA takes work items
// (unit, head block) round-robin.  Warp NW is the producer: its lane 0 streams
// the unit's pages into a ring of shared-memory stages with 1-D bulk copies
// (cp.async.bulk, completion on an mbarrier).  Warps 0..NW-1 consume: scores
// by FMA + warp-shuffle reduction, online softmax in the log2 domain, and the
// running output in registers.  The ring keeps several pages in flight per SM.
#include "common.cuh"
#include "finish.cuh"
#include "kernels.h"

namespace dcp {

namespace {

constexpr int kNW = 4;                 // consumer warps
constexpr int kThreads = 32 * (kNW + 1);

struct Ring {
    uint64_t* full;
    uint64_t* empty;
    int stages;
};

// Producer-side bounded drain: wait for copies still in flight before exit.
__device__ void drain_ring(const Ring& r, int stage, uint32_t phase, int issued, int* status) {
    int n = issued < r.stages ? issued : r.stages;
    for (int k = 0; k < n; k++) {
        stage = stage == 0 ? r.stages - 1 : stage - 1;
        if (stage == r.stages - 1) phase ^= 1;
        mbar_wait(r.full + stage, phase, nullptr, status);
    }
}

// ---------------------------------------------------------------------------
// GQA: item = (unit, kv head g); G query heads per kv head; head dim D.
// Lanes of a warp split a row into 16-byte chunks (D/8 lanes per row); a warp
// covers 256/D rows per pass.
// ---------------------------------------------------------------------------
template <int D, int G>
__global__ void __launch_bounds__(kThreads) gqa_simt_kernel(DecodeArgs a, int stages) {
    constexpr int LPR = D / 8;
    constexpr int R = 32 / LPR;
    constexpr int RG = kNW * R;  // row groups per CTA
    extern __shared__ __align__(128) uint8_t smem[];
    const int P = a.page_size;
    const uint32_t blk_bytes = (uint32_t)P * D * 2;
    uint8_t* sK = smem;
    uint8_t* sV = sK + (size_t)stages * blk_bytes;
    float* cm = reinterpret_cast<float*>(sV + (size_t)stages * blk_bytes);
    float* cl = cm + RG * G;
    float* cacc = cl + RG * G;            // [RG][G][D]
    float* sO = cacc + RG * G * D;        // [G][D]
    float* sLse = sO + G * D;             // [G]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sLse + 32);
    Ring ring{bars, bars + stages, stages};
    __shared__ int s_flag;
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; s++) {
            mbar_init(ring.full + s, 1);
            mbar_init(ring.empty + s, kNW);
        }
        s_abort = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int n_hb = a.hkv;
    const int num_items = a.plan->num_units * n_hb;

    if (warp == kNW) {
        if (lane != 0) return;
        int stage = 0, issued = 0;
        uint32_t phase = 0;
        const uint64_t pol = l2_policy_evict_first();
        for (int item = blockIdx.x; item < num_items && !s_abort; item += gridDim.x) {
            const Unit u = a.units[item / n_hb];
            const int g = item % n_hb;
            const int j0 = u.t0 / P, j1 = (u.t1 + P - 1) / P;
            for (int j = j0; j < j1; j++) {
                if (!mbar_wait(ring.empty + stage, phase ^ 1, &s_abort, a.status)) break;
                const int pg = page_of(a, u.n, u.b, j);
                if (pg >= 0) {
                    mbar_arrive_expect_tx(ring.full + stage, 2 * blk_bytes);
                    const int64_t off = (((int64_t)pg * a.hkv + g) * P) * D * 2;
                    bulk_g2s_hint(sK + (size_t)stage * blk_bytes, a.k_pages + off, blk_bytes, ring.full + stage, pol);
                    bulk_g2s_hint(sV + (size_t)stage * blk_bytes, a.v_pages + off, blk_bytes, ring.full + stage, pol);
                } else {
                    record_status(a.status, DCP_ERR_UNALLOCATED_PAGE);
                    mbar_arrive(ring.full + stage);
                }
                issued++;
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        if (s_abort) drain_ring(ring, stage, phase, issued, a.status);
        return;
    }

    // consumers
    const int rin = lane / LPR;      // row within this warp's pass
    const int ch = lane % LPR;       // 16-byte chunk of the row
    const int rg = warp * R + rin;   // row group id
    int stage = 0;
    uint32_t phase = 0;
    for (int item = blockIdx.x; item < num_items; item += gridDim.x) {
        const Unit u = a.units[item / n_hb];
        const int g = item % n_hb;
        float q[G][8];
        {
            const __nv_bfloat16* qb = a.q + ((int64_t)u.b * a.hq + g * G) * D + ch * 8;
#pragma unroll
            for (int h = 0; h < G; h++) {
                uint4 w = *reinterpret_cast<const uint4*>(qb + (int64_t)h * D);
                uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    q[h][2 * e] = bf16_lo(ws[e]) * a.scale_log2;
                    q[h][2 * e + 1] = bf16_hi(ws[e]) * a.scale_log2;
                }
            }
        }
        float m[G], l[G], acc[G][8];
#pragma unroll
        for (int h = 0; h < G; h++) {
            m[h] = -INFINITY;
            l[h] = 0.f;
#pragma unroll
            for (int e = 0; e < 8; e++) acc[h][e] = 0.f;
        }
        const int j0 = u.t0 / P, j1 = (u.t1 + P - 1) / P;
        bool ok = true;
        for (int j = j0; j < j1; j++) {
            if (!mbar_wait(ring.full + stage, phase, &s_abort, a.status)) {
                ok = false;
                break;
            }
            const int pg = page_of(a, u.n, u.b, j);
            const int rhi = min(u.t1 - j * P, P);
            if (pg >= 0) {
                const uint8_t* kb = sK + (size_t)stage * blk_bytes;
                const uint8_t* vb = sV + (size_t)stage * blk_bytes;
                for (int r0 = warp * R; r0 < P; r0 += RG) {
                    const int r = r0 + rin;
                    uint4 kw = *reinterpret_cast<const uint4*>(kb + ((size_t)r * D + ch * 8) * 2);
                    uint4 vw = *reinterpret_cast<const uint4*>(vb + ((size_t)r * D + ch * 8) * 2);
                    float kf[8], vf[8];
                    uint32_t kws[4] = {kw.x, kw.y, kw.z, kw.w}, vws[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        kf[2 * e] = bf16_lo(kws[e]);
                        kf[2 * e + 1] = bf16_hi(kws[e]);
                        vf[2 * e] = bf16_lo(vws[e]);
                        vf[2 * e + 1] = bf16_hi(vws[e]);
                    }
                    const bool valid = r < rhi;
#pragma unroll
                    for (int h = 0; h < G; h++) {
                        float s = 0.f;
#pragma unroll
                        for (int e = 0; e < 8; e++) s = fmaf(q[h][e], kf[e], s);
#pragma unroll
                        for (int o = 1; o < LPR; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                        if (valid) {
                            const float mn = fmaxf(m[h], s);
                            const float corr = fast_exp2(m[h] - mn);
                            const float p = fast_exp2(s - mn);
                            m[h] = mn;
                            l[h] = l[h] * corr + p;
#pragma unroll
                            for (int e = 0; e < 8; e++) acc[h][e] = fmaf(p, vf[e], acc[h][e] * corr);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(ring.empty + stage);
            if (++stage == stages) {
                stage = 0;
                phase ^= 1;
            }
        }
        if (!ok) break;
        // combine the row groups of all consumer warps
#pragma unroll
        for (int h = 0; h < G; h++) {
            if (ch == 0) {
                cm[rg * G + h] = m[h];
                cl[rg * G + h] = l[h];
            }
#pragma unroll
            for (int e = 0; e < 8; e++) cacc[(rg * G + h) * D + ch * 8 + e] = acc[h][e];
        }
        named_barrier_sync(1, kNW * 32);
        const int tid = threadIdx.x;
        for (int i = tid; i < G * D; i += kNW * 32) {
            const int h = i / D, d = i - h * D;
            float M = -INFINITY;
            for (int k = 0; k < RG; k++) M = fmaxf(M, cm[k * G + h]);
            float o = 0.f, ls = 0.f;
            if (M != -INFINITY) {
                for (int k = 0; k < RG; k++) {
                    const float w = fast_exp2(cm[k * G + h] - M);
                    ls += cl[k * G + h] * w;
                    o += cacc[(k * G + h) * D + d] * w;
                }
                o /= ls;
            }
            sO[i] = o;
            if (d == 0) sLse[h] = (M == -INFINITY) ? -INFINITY : (M + log2f(ls)) * kLn2;
        }
        named_barrier_sync(1, kNW * 32);
        finish_unit<kNW * 32>(a, u, g, n_hb, g * G, G, sO, sLse, &s_flag, tid, 1);
        named_barrier_sync(1, kNW * 32);
    }
}

// ---------------------------------------------------------------------------
// MLA: item = (unit, block of 16 query heads); each consumer warp owns 4
// heads and every row of the stage.  A stage is 16 consecutive tokens of one
// page (bf16: 18 KB; fp8: 9 KB + 64 B of scales).  Lanes split a row into
// 8-element chunks: lane owns chunks lane, lane+32, lane+64 (< 72); the value
// (first 512 entries) is chunks lane and lane+32.
// ---------------------------------------------------------------------------
constexpr int kMlaRows = 16;
constexpr int kMlaHeadsPerWarp = 4;
constexpr int kMlaHeadBlock = kNW * kMlaHeadsPerWarp;

template <bool FP8>
__global__ void __launch_bounds__(kThreads) mla_simt_kernel(DecodeArgs a, int stages) {
    constexpr int DK = 576, DV = 512, NCH = DK / 8;
    constexpr int ELT = FP8 ? 1 : 2;
    constexpr uint32_t kRowBytes = DK * ELT;
    constexpr uint32_t kStageBytes = kMlaRows * kRowBytes;
    extern __shared__ __align__(128) uint8_t smem[];
    const int P = a.page_size;
    uint8_t* sRows = smem;
    float* sScale = reinterpret_cast<float*>(sRows + (size_t)stages * kStageBytes);  // [stages][16]
    float* sO = sScale + stages * kMlaRows;                                          // [16][512]
    float* sLse = sO + kMlaHeadBlock * DV;                                           // [16]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sLse + 32);
    Ring ring{bars, bars + stages, stages};
    __shared__ int s_flag;
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; s++) {
            mbar_init(ring.full + s, 1);
            mbar_init(ring.empty + s, kNW);
        }
        s_abort = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int n_hb = a.hq / kMlaHeadBlock;
    const int num_items = a.plan->num_units * n_hb;
    const int sub_per_page = P / kMlaRows;

    if (warp == kNW) {
        if (lane != 0) return;
        int stage = 0, issued = 0;
        uint32_t phase = 0;
        const uint64_t pol = l2_policy_evict_first();
        for (int item = blockIdx.x; item < num_items && !s_abort; item += gridDim.x) {
            const Unit u = a.units[item / n_hb];
            const int r0 = u.t0, r1 = u.t1;
            for (int t = r0; t < r1; t += kMlaRows) {
                if (!mbar_wait(ring.empty + stage, phase ^ 1, &s_abort, a.status)) break;
                const int j = t / P, sub = (t % P) / kMlaRows;
                const int pg = page_of(a, u.n, u.b, j);
                if (pg >= 0) {
                    const int64_t row0 = (int64_t)pg * P + sub * kMlaRows;
                    mbar_arrive_expect_tx(ring.full + stage, kStageBytes + (FP8 ? kMlaRows * 4 : 0));
                    bulk_g2s_hint(sRows + (size_t)stage * kStageBytes, a.k_pages + row0 * kRowBytes, kStageBytes,
                                  ring.full + stage, pol);
                    if (FP8)
                        bulk_g2s(sScale + stage * kMlaRows, a.kv_scales + row0, kMlaRows * 4, ring.full + stage);
                } else {
                    record_status(a.status, DCP_ERR_UNALLOCATED_PAGE);
                    mbar_arrive(ring.full + stage);
                }
                issued++;
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        (void)sub_per_page;
        if (s_abort) drain_ring(ring, stage, phase, issued, a.status);
        return;
    }

    int stage = 0;
    uint32_t phase = 0;
    for (int item = blockIdx.x; item < num_items; item += gridDim.x) {
        const Unit u = a.units[item / n_hb];
        const int hb = item % n_hb;
        const int hw0 = hb * kMlaHeadBlock + warp * kMlaHeadsPerWarp;  // first head of this warp
        float q[kMlaHeadsPerWarp][3][8];
#pragma unroll
        for (int h = 0; h < kMlaHeadsPerWarp; h++) {
            const __nv_bfloat16* qh = a.q + ((int64_t)u.b * a.hq + hw0 + h) * DK;
#pragma unroll
            for (int c = 0; c < 3; c++) {
                const int chn = lane + 32 * c;
                if (chn < NCH) {
                    uint4 w = *reinterpret_cast<const uint4*>(qh + chn * 8);
                    uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        q[h][c][2 * e] = bf16_lo(ws[e]) * a.scale_log2;
                        q[h][c][2 * e + 1] = bf16_hi(ws[e]) * a.scale_log2;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; e++) q[h][c][e] = 0.f;
                }
            }
        }
        float m[kMlaHeadsPerWarp], l[kMlaHeadsPerWarp], acc[kMlaHeadsPerWarp][2][8];
#pragma unroll
        for (int h = 0; h < kMlaHeadsPerWarp; h++) {
            m[h] = -INFINITY;
            l[h] = 0.f;
#pragma unroll
            for (int c = 0; c < 2; c++)
#pragma unroll
                for (int e = 0; e < 8; e++) acc[h][c][e] = 0.f;
        }
        bool ok = true;
        for (int t = u.t0; t < u.t1; t += kMlaRows) {
            if (!mbar_wait(ring.full + stage, phase, &s_abort, a.status)) {
                ok = false;
                break;
            }
            const int j = t / P;
            const int pg = page_of(a, u.n, u.b, j);
            const int nrows = min(u.t1 - t, kMlaRows);
            if (pg >= 0) {
                const uint8_t* rows = sRows + (size_t)stage * kStageBytes;
                for (int r = 0; r < nrows; r++) {
                    const uint8_t* row = rows + (size_t)r * kRowBytes;
                    float x[3][8];
#pragma unroll
                    for (int c = 0; c < 3; c++) {
                        const int chn = lane + 32 * c;
                        if (chn < NCH) {
                            if (FP8) {
                                uint2 w = *reinterpret_cast<const uint2*>(row + chn * 8);
                                uint32_t ws[2] = {w.x, w.y};
#pragma unroll
                                for (int e = 0; e < 2; e++) {
                                    float2 f0 = e4m3x2_to_float2((uint16_t)(ws[e] & 0xFFFF));
                                    float2 f1 = e4m3x2_to_float2((uint16_t)(ws[e] >> 16));
                                    x[c][4 * e] = f0.x;
                                    x[c][4 * e + 1] = f0.y;
                                    x[c][4 * e + 2] = f1.x;
                                    x[c][4 * e + 3] = f1.y;
                                }
                            } else {
                                uint4 w = *reinterpret_cast<const uint4*>(row + chn * 16);
                                uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                                for (int e = 0; e < 4; e++) {
                                    x[c][2 * e] = bf16_lo(ws[e]);
                                    x[c][2 * e + 1] = bf16_hi(ws[e]);
                                }
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; e++) x[c][e] = 0.f;
                        }
                    }
                    const float ts = FP8 ? sScale[stage * kMlaRows + r] : 1.f;
#pragma unroll
                    for (int h = 0; h < kMlaHeadsPerWarp; h++) {
                        float s = 0.f;
#pragma unroll
                        for (int c = 0; c < 3; c++)
#pragma unroll
                            for (int e = 0; e < 8; e++) s = fmaf(q[h][c][e], x[c][e], s);
#pragma unroll
                        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                        s *= ts;
                        const float mn = fmaxf(m[h], s);
                        const float corr = fast_exp2(m[h] - mn);
                        const float p = fast_exp2(s - mn);
                        m[h] = mn;
                        l[h] = l[h] * corr + p;
                        const float pv = p * ts;
#pragma unroll
                        for (int c = 0; c < 2; c++)
#pragma unroll
                            for (int e = 0; e < 8; e++) acc[h][c][e] = fmaf(pv, x[c][e], acc[h][c][e] * corr);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(ring.empty + stage);
            if (++stage == stages) {
                stage = 0;
                phase ^= 1;
            }
        }
        if (!ok) break;
#pragma unroll
        for (int h = 0; h < kMlaHeadsPerWarp; h++) {
            const int hl = warp * kMlaHeadsPerWarp + h;
            const float inv = l[h] > 0.f ? 1.f / l[h] : 0.f;
#pragma unroll
            for (int c = 0; c < 2; c++)
#pragma unroll
                for (int e = 0; e < 8; e++) sO[hl * DV + (lane + 32 * c) * 8 + e] = acc[h][c][e] * inv;
            if (lane == 0) sLse[hl] = (m[h] == -INFINITY) ? -INFINITY : (m[h] + log2f(l[h])) * kLn2;
        }
        named_barrier_sync(1, kNW * 32);
        finish_unit<kNW * 32>(a, u, hb, n_hb, hb * kMlaHeadBlock, kMlaHeadBlock, sO, sLse, &s_flag, threadIdx.x, 1);
        named_barrier_sync(1, kNW * 32);
    }
}

template <int D, int G>
size_t gqa_smem(int P, int stages) {
    constexpr int R = 32 / (D / 8);
    constexpr int RG = kNW * R;
    return (size_t)stages * 2 * P * D * 2 + (size_t)(2 * RG * G + RG * G * D + G * D + 32) * 4 +
           (size_t)stages * 2 * 8;
}

size_t mla_smem(bool fp8, int stages) {
    const size_t stage_bytes = (size_t)kMlaRows * 576 * (fp8 ? 1 : 2);
    return (size_t)stages * stage_bytes + (size_t)stages * kMlaRows * 4 + (size_t)(kMlaHeadBlock * 512 + 32) * 4 +
           (size_t)stages * 2 * 8;
}

template <int D, int G>
int gqa_stages(int P) {
    // ring of 2..6 pages within ~180 KB of shared memory
    const size_t fixed = gqa_smem<D, G>(P, 0);
    const size_t per = (size_t)2 * P * D * 2 + 16;
    size_t n = (180 * 1024 - fixed) / per;
    return (int)(n < 2 ? 2 : (n > 6 ? 6 : n));
}

template <int D, int G>
cudaError_t run_gqa(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s) {
    const int stages = gqa_stages<D, G>(a.page_size);
    const size_t smem = gqa_smem<D, G>(a.page_size, stages);
    cudaError_t e = cudaFuncSetAttribute(gqa_simt_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    gqa_simt_kernel<D, G><<<g.ctas, kThreads, smem, s>>>(a, stages);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_simt(const DecodeGeometry& g, const DecodeArgs& a, cudaStream_t s) {
    if (g.path == DecodePath::GqaSimt) {
        const int G = a.hq / a.hkv;
#define DCP_GQA_CASE(DD, GG) \
    if (a.dk == DD && G == GG) return run_gqa<DD, GG>(g, a, s);
        DCP_GQA_CASE(64, 1) DCP_GQA_CASE(64, 2) DCP_GQA_CASE(64, 4) DCP_GQA_CASE(64, 8)
        DCP_GQA_CASE(128, 1) DCP_GQA_CASE(128, 2) DCP_GQA_CASE(128, 4) DCP_GQA_CASE(128, 8)
#undef DCP_GQA_CASE
        return cudaErrorNotSupported;
    }
    if (g.path == DecodePath::MlaSimt) {
        const bool fp8 = a.kv_scales != nullptr;
        const int stages = 4;
        const size_t smem = mla_smem(fp8, stages);
        cudaError_t e;
        if (fp8) {
            e = cudaFuncSetAttribute(mla_simt_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            mla_simt_kernel<true><<<g.ctas, kThreads, smem, s>>>(a, stages);
        } else {
            e = cudaFuncSetAttribute(mla_simt_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            mla_simt_kernel<false><<<g.ctas, kThreads, smem, s>>>(a, stages);
        }
        return cudaGetLastError();
    }
    return cudaErrorNotSupported;
}

// Resident CTAs per SM of the kernel a launch with these parameters would use.
int simt_blocks_per_sm(DecodePath p, int D, int G, int P, bool fp8) {
    const void* fn = nullptr;
    if (p == DecodePath::MlaSimt) {
        fn = fp8 ? (const void*)mla_simt_kernel<true> : (const void*)mla_simt_kernel<false>;
    } else {
#define DCP_FN_CASE(DD, GG) \
    if (D == DD && G == GG) fn = (const void*)gqa_simt_kernel<DD, GG>;
        DCP_FN_CASE(64, 1) DCP_FN_CASE(64, 2) DCP_FN_CASE(64, 4) DCP_FN_CASE(64, 8)
        DCP_FN_CASE(128, 1) DCP_FN_CASE(128, 2) DCP_FN_CASE(128, 4) DCP_FN_CASE(128, 8)
#undef DCP_FN_CASE
    }
    if (!fn) return 0;
    const size_t smem = simt_smem_bytes(p, D, G, P, fp8);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, smem) != cudaSuccess) return 0;
    return n;
}

size_t simt_smem_bytes(DecodePath p, int D, int G, int P, bool fp8) {
    if (p == DecodePath::MlaSimt) return mla_smem(fp8, 4);
#define DCP_SMEM_CASE(DD, GG) \
    if (D == DD && G == GG) return gqa_smem<DD, GG>(P, gqa_stages<DD, GG>(P));
    DCP_SMEM_CASE(64, 1) DCP_SMEM_CASE(64, 2) DCP_SMEM_CASE(64, 4) DCP_SMEM_CASE(64, 8)
    DCP_SMEM_CASE(128, 1) DCP_SMEM_CASE(128, 2) DCP_SMEM_CASE(128, 4) DCP_SMEM_CASE(128, 8)
#undef DCP_SMEM_CASE
    return 0;
}

}  // namespace dcp
