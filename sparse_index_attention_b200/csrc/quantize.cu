// quantize.cu -- cache-write quantizers: bf16/fp32 rows -> FP8 E4M3 codes + fp32 group scales,
// scattered to their physical cache slots ("Day 0 Inference Adaptation and Optimization for
// Hybrid Attention Models", "Hierarchical Quantization"; "Inference Adaptation and Performance
// Optimization for a Domestically Developed LLM's New Architecture", section 4 table: dynamic
// per-group scales for the index keys, per-token tiles for the latent KV cache).
//
// Scale rule (dynamic max-abs): scale = amax / 448, inv = 448 / amax, both IEEE fp32 round to
// nearest (this file is built without fast-math, so `/` is the correctly rounded division);
// code = cvt.rn.satfinite to E4M3 of x * inv.  An all-zero group gets scale 1 and code 0.
#include "kernels.h"

namespace hsa {

namespace {

constexpr int kThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kThreads)
quantize_groups_kernel(const T* __restrict__ src, int64_t n_rows, int src_stride, int D, int group,
                       const int64_t* __restrict__ slot_mapping, int64_t num_slots,
                       uint8_t* __restrict__ codes, float* __restrict__ scales) {
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int ng = D / group;
    if (warp >= n_rows * ng) return;
    const int64_t r = warp / ng;
    const int g = (int)(warp % ng);
    const int64_t slot = slot_mapping ? slot_mapping[r] : r;
    if (slot < 0 || slot >= num_slots) return;
    const T* x = src + r * src_stride + (int64_t)g * group;
    float amax = 0.f;
    for (int i = lane; i < group; i += 32) amax = fmaxf(amax, fabsf(to_f32(x[i])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float scale = 1.f, inv = 0.f;
    if (amax > 0.f) {
        scale = amax / 448.0f;
        inv = 448.0f / amax;
    }
    if (lane == 0) scales[slot * ng + g] = scale;
    uint8_t* c = codes + slot * D + (int64_t)g * group;
    for (int i = lane; i < group; i += 32) {
        const float y = __fmul_rn(to_f32(x[i]), inv);
        c[i] = amax > 0.f ? (uint8_t)__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3) : (uint8_t)0;
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
copy_cols_kernel(const T* __restrict__ src, int64_t n_rows, int src_stride, int col0, int cols,
                 const int64_t* __restrict__ slot_mapping, int64_t num_slots,
                 __nv_bfloat16* __restrict__ dst) {
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= n_rows * cols) return;
    const int64_t r = i / cols;
    const int c = (int)(i % cols);
    const int64_t slot = slot_mapping ? slot_mapping[r] : r;
    if (slot < 0 || slot >= num_slots) return;
    dst[slot * cols + c] = __float2bfloat16(to_f32(src[r * src_stride + col0 + c]));
}

template <typename T>
cudaError_t launch_t(const void* src, int64_t n_rows, int32_t src_stride, int32_t D, int32_t group,
                     const int64_t* slot_mapping, int64_t num_slots, uint8_t* codes, float* scales,
                     int32_t copy_cols, void* copy_dst, cudaStream_t st) {
    const int64_t warps = n_rows * (D / group);
    const int64_t blocks = ceil_div(warps * 32, kThreads);
    quantize_groups_kernel<T><<<(unsigned)blocks, kThreads, 0, st>>>(
        reinterpret_cast<const T*>(src), n_rows, src_stride, D, group, slot_mapping, num_slots,
        codes, scales);
    count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || copy_cols == 0) return e;
    const int64_t n = n_rows * copy_cols;
    copy_cols_kernel<T><<<(unsigned)ceil_div(n, kThreads), kThreads, 0, st>>>(
        reinterpret_cast<const T*>(src), n_rows, src_stride, D, copy_cols, slot_mapping, num_slots,
        reinterpret_cast<__nv_bfloat16*>(copy_dst));
    count_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_rows(const void* src, hsa_dtype_t src_dtype, int64_t n_rows,
                                 int32_t src_stride, int32_t D, int32_t group,
                                 const int64_t* slot_mapping, int64_t num_slots, uint8_t* codes,
                                 float* scales, int32_t copy_cols, void* copy_dst,
                                 cudaStream_t st) {
    if (n_rows == 0) return cudaSuccess;
    if (src_dtype == HSA_F32)
        return launch_t<float>(src, n_rows, src_stride, D, group, slot_mapping, num_slots, codes,
                               scales, copy_cols, copy_dst, st);
    return launch_t<__nv_bfloat16>(src, n_rows, src_stride, D, group, slot_mapping, num_slots, codes,
                                   scales, copy_cols, copy_dst, st);
}

}  // namespace hsa
