// synth_fill.cu -- device-side fill of the seeded synthetic inputs.
//
// Builds libsynth.so.  The kernels evaluate the counter-based generator of
// synth_hash.h on the GPU so that multi-gigabyte inputs need not cross PCIe;
// the bits equal the host (numpy / C) evaluation of the same definition.
// Nothing here belongs to the attention method.
#include <cuda_runtime.h>
#include <stdint.h>

#include "synth_hash.h"

namespace {

__global__ void fill_flat_kernel(uint16_t* __restrict__ out, int64_t n, uint64_t key) {
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        out[i] = synth_bf16_at(key, (uint64_t)i);
}

// out[r][g][d] = bf16 of stream `key` at synth_kv_index(req[r], pos[r], g, d, hkv, w)
__global__ void fill_kv_rows_kernel(uint16_t* __restrict__ out, int64_t n_rows,
                                    const int32_t* __restrict__ req, const int32_t* __restrict__ pos,
                                    int hkv, int w, uint64_t key) {
    int64_t total = n_rows * (int64_t)hkv * w;
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        int64_t r = i / ((int64_t)hkv * w);
        int rem = (int)(i - r * (int64_t)hkv * w);
        int g = rem / w;
        int d = rem - g * w;
        uint64_t idx = synth_kv_index((uint64_t)req[r], (uint64_t)pos[r], (uint64_t)g, (uint64_t)d,
                                      (uint64_t)hkv, (uint64_t)w);
        out[i] = synth_bf16_at(key, idx);
    }
}

int grid_for(int64_t n) {
    int64_t g = (n + 255) / 256;
    if (g > 148 * 32) g = 148 * 32;
    if (g < 1) g = 1;
    return (int)g;
}

}  // namespace

extern "C" {

// Fill out[0..n) (bf16 bits) with stream `key` at flat indices 0..n-1.
int synth_fill_flat(void* out, int64_t n, uint64_t key, void* stream) {
    if (n < 0 || (n > 0 && out == nullptr)) return 1;
    if (n == 0) return 0;
    fill_flat_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((uint16_t*)out, n, key);
    return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

// Fill rows [n_rows][hkv][w] (bf16 bits) for (req[r], pos[r]) pairs (device int32 arrays).
int synth_fill_kv_rows(void* out, int64_t n_rows, const void* req, const void* pos, int32_t hkv,
                       int32_t w, uint64_t key, void* stream) {
    if (n_rows < 0 || hkv < 1 || w < 1) return 1;
    if (n_rows == 0) return 0;
    if (!out || !req || !pos) return 1;
    fill_kv_rows_kernel<<<grid_for(n_rows * (int64_t)hkv * w), 256, 0, (cudaStream_t)stream>>>(
        (uint16_t*)out, n_rows, (const int32_t*)req, (const int32_t*)pos, hkv, w, key);
    return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

}  // extern "C"
