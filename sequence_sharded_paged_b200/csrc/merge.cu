// merge.cu -- LSE-weighted merge of the N shard partials (dcp_merge).
//
// "Efficient Decode Context Parallelism with vLLM for Long Context Workloads",
// section 4.1: the all-gathered LSE values reweight the partial outputs and
// the reduce-scatter sums them.  With every shard on one GPU the same
// arithmetic is one pass over o_partial:
//   M = max_n lse_n,  LSE = M + ln sum_n exp(lse_n - M),
//   out = sum_n exp(lse_n - LSE) * o_n.
// HBM-bound: one warp per (b, h) row streams the N rows with 16-byte loads.
#include "common.cuh"
#include "kernels.h"

namespace dcp {

namespace {

constexpr int kMergeWarps = 8;
constexpr int kMergeFast = 8;  // shard counts up to this take the path with all loads in flight

__global__ void __launch_bounds__(32 * kMergeWarps)
    merge_kernel(int N, int64_t BH, int Dv, const float* __restrict__ o_part, const float* __restrict__ lse_part,
                 float* __restrict__ out, float* __restrict__ lse_out, int discard) {
    const int64_t row = (int64_t)blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= BH) return;
    float M = -INFINITY;
    for (int n = 0; n < N; n++) M = fmaxf(M, __ldg(lse_part + (int64_t)n * BH + row));
    float4* o = reinterpret_cast<float4*>(out + row * Dv);
    const int nv = Dv / 4;
    if (M == -INFINITY) {
        for (int v = lane; v < nv; v += 32) o[v] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lane == 0 && lse_out) lse_out[row] = -INFINITY;
        return;
    }
    float sum = 0.f;
    for (int n = 0; n < N; n++) sum += expf(__ldg(lse_part + (int64_t)n * BH + row) - M);
    const float L = M + logf(sum);
    if (lane == 0 && lse_out) lse_out[row] = L;
    if (N <= kMergeFast) {
        // the row's weights once, then every shard's 16 bytes of a column block loaded before any
        // is used, so that N loads per lane are in flight (a shard with weight 0 is not read)
        float w[kMergeFast];
#pragma unroll
        for (int n = 0; n < kMergeFast; n++) {
            const float ln = n < N ? __ldg(lse_part + (int64_t)n * BH + row) : -INFINITY;
            w[n] = ln == -INFINITY ? 0.f : expf(ln - L);
        }
        for (int v = lane; v < nv; v += 32) {
            float4 x[kMergeFast];
#pragma unroll
            for (int n = 0; n < kMergeFast; n++)
                x[n] = w[n] != 0.f
                           ? __ldcs(reinterpret_cast<const float4*>(o_part + ((int64_t)n * BH + row) * Dv) + v)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int n = 0; n < kMergeFast; n++) {
                if (w[n] == 0.f) continue;
                acc.x = fmaf(w[n], x[n].x, acc.x);
                acc.y = fmaf(w[n], x[n].y, acc.y);
                acc.z = fmaf(w[n], x[n].z, acc.z);
                acc.w = fmaf(w[n], x[n].w, acc.w);
            }
            o[v] = acc;
        }
    } else {
        for (int v = lane; v < nv; v += 32) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int n = 0; n < N; n++) {
                const float ln = __ldg(lse_part + (int64_t)n * BH + row);
                if (ln == -INFINITY) continue;
                const float w = expf(ln - L);
                const float4 x = __ldcs(reinterpret_cast<const float4*>(o_part + ((int64_t)n * BH + row) * Dv) + v);
                acc.x = fmaf(w, x.x, acc.x);
                acc.y = fmaf(w, x.y, acc.y);
                acc.z = fmaf(w, x.z, acc.z);
                acc.w = fmaf(w, x.w, acc.w);
            }
            o[v] = acc;
        }
    }
    if (discard) {  // the partials are scratch: drop their lines from L2 without writing them back
        __syncwarp();
        for (int i = lane; i < N * (Dv / 32); i += 32) {
            const int n = i / (Dv / 32), l = i - n * (Dv / 32);
            discard_l2_line(o_part + ((int64_t)n * BH + row) * Dv + l * 32);
        }
    }
}

// One rank's share of the merge across GPUs, between the all-gather of the
// LSEs and the reduce-scatter of the outputs: with every shard's LSE of row
// (b, h) at hand, LSE = M + ln sum_n exp(lse_n - M), and this rank's partial
// enters the sum with weight exp(lse_rank - LSE).  The weighted row goes to the
// reduce-scatter layout [N][B][H/N][Dv] (block n holds the heads rank n keeps).
__global__ void __launch_bounds__(32 * kMergeWarps)
    lse_rescale_kernel(int N, int rank, int B, int H, int Dv, const float* __restrict__ lse_all,
                       const float* __restrict__ o, float* __restrict__ o_rs, float* __restrict__ lse_out) {
    const int64_t BH = (int64_t)B * H;
    const int64_t row = (int64_t)blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= BH) return;
    float M = -INFINITY;
    for (int n = 0; n < N; n++) M = fmaxf(M, __ldg(lse_all + (int64_t)n * BH + row));
    float L = -INFINITY, w = 0.f;
    if (M != -INFINITY) {
        float sum = 0.f;
        for (int n = 0; n < N; n++) sum += expf(__ldg(lse_all + (int64_t)n * BH + row) - M);
        L = M + logf(sum);
        const float lr = __ldg(lse_all + (int64_t)rank * BH + row);
        w = lr == -INFINITY ? 0.f : expf(lr - L);
    }
    if (lane == 0 && lse_out) lse_out[row] = L;
    const int b = (int)(row / H), h = (int)(row - (int64_t)b * H);
    const int Hn = H / N;
    const float4* src = reinterpret_cast<const float4*>(o + row * Dv);
    float4* dst = reinterpret_cast<float4*>(o_rs + (((int64_t)(h / Hn) * B + b) * Hn + h % Hn) * Dv);
    for (int v = lane; v < Dv / 4; v += 32) {
        const float4 x = __ldg(src + v);
        dst[v] = make_float4(w * x.x, w * x.y, w * x.z, w * x.w);
    }
}

}  // namespace

cudaError_t launch_lse_rescale(int N, int rank, int B, int H, int Dv, const float* lse_all, const float* o,
                               float* o_rs, float* lse_out, cudaStream_t s) {
    const int64_t BH = (int64_t)B * H;
    const int64_t blocks = (BH + kMergeWarps - 1) / kMergeWarps;
    lse_rescale_kernel<<<(unsigned)blocks, 32 * kMergeWarps, 0, s>>>(N, rank, B, H, Dv, lse_all, o, o_rs, lse_out);
    return cudaGetLastError();
}

cudaError_t launch_merge(int N, int B, int H, int Dv, const float* o_partial, const float* lse, float* out,
                         float* lse_out, bool discard, cudaStream_t s) {
    const int64_t BH = (int64_t)B * H;
    const int64_t blocks = (BH + kMergeWarps - 1) / kMergeWarps;
    merge_kernel<<<(unsigned)blocks, 32 * kMergeWarps, 0, s>>>(N, BH, Dv, o_partial, lse, out, lse_out,
                                                                discard && Dv % 32 == 0 ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace dcp
