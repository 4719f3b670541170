// quantize.cu -- cache-write quantizers: bf16/fp32 rows -> FP8 E4M3 codes + fp32 group scales,
// scattered to their physical cache slots ("Day 0 Inference Adaptation and Optimization for
// Hybrid Attention Models", "Hierarchical Quantization"; "Inference Adaptation and Performance
// Optimization for a Domestically Developed LLM's New Architecture", section 4 table: dynamic
// per-group scales for the index keys, per-token tiles for the latent KV cache).
//
// Scale rule (dynamic max-abs): scale = amax / 448, inv = 448 / amax, both IEEE fp32 round to
// nearest (this file is built without fast-math, so `/` is the correctly rounded division);
// code = cvt.rn.satfinite to E4M3 of x * inv.  An all-zero group gets scale 1 and code 0.  A
// group maximum below 2^-64 is lifted by 2^64 together with the values before inv and the
// products are formed, so inv stays finite.
//
// MXFP8 (the pages' format for the index Q/K): 32-element blocks share one E8M0 byte E = X + 127,
// X = floor(log2(amax)) - 8 clamped to [-127, 127]; the codes are E4M3 of x * 2^-X.
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
    // below 2^-64 the maximum and the values are lifted by 2^64 (exact) first: 448 / amax would
    // overflow for amax < 448 / FLT_MAX and turn the group's zeros into 0 * inf = NaN; where it
    // is finite the lift changes no code (reciprocal and products move by a power of two)
    const float lift = amax < 0x1p-64f ? 0x1p64f : 1.f;
    float scale = 1.f, inv = 0.f;
    if (amax > 0.f) {
        scale = amax / 448.0f;
        inv = 448.0f / (amax * lift);
    }
    if (lane == 0) scales[slot * ng + g] = scale;
    uint8_t* c = codes + slot * D + (int64_t)g * group;
    for (int i = lane; i < group; i += 32) {
        const float y = __fmul_rn(__fmul_rn(to_f32(x[i]), lift), inv);
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

// floor(log2(a)) of a positive finite float, from its bits (subnormals included).
__device__ __forceinline__ int floor_log2(float a) {
    const uint32_t bits = __float_as_uint(a);
    const int e = (int)(bits >> 23);
    if (e) return e - 127;
    return (31 - __clz((int)(bits & 0x7FFFFFu))) - 149;
}

// MXFP8 ("Day 0 Inference Adaptation and Optimization for Hybrid Attention Models",
// "Hierarchical Quantization": index Q/K in blocks of 32 sharing one exponent).
// One warp per 32-element block, one element per lane.  X = floor(log2(amax)) - 8
// clamped to [-127, 127]; the element is x * 2^-X (a power-of-two rescale, exact whenever the
// result is at least 2^-126, and below that every candidate rounds to code 0) rounded to E4M3.
template <typename T>
__global__ void __launch_bounds__(kThreads)
quantize_mx_kernel(const T* __restrict__ src, int64_t n_rows, int D,
                   const int64_t* __restrict__ slot_mapping, int64_t num_slots,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int nb = D / 32;
    if (warp >= n_rows * nb) return;
    const int64_t r = warp / nb;
    const int b = (int)(warp % nb);
    const int64_t slot = slot_mapping ? slot_mapping[r] : r;
    if (slot < 0 || slot >= num_slots) return;
    const float x = to_f32(src[r * D + (int64_t)b * 32 + lane]);
    float amax = fabsf(x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    uint8_t code = 0;
    int E = 0;
    if (amax > 0.f) {
        const int X = min(127, max(-127, floor_log2(amax) - 8));
        E = X + 127;
        // 2^-X: X lies in [-127, 119] (amax <= FLT_MAX), so the exponent field 127 - X lies in
        // [8, 254] and the power of two is a normal float
        const float inv = __uint_as_float((uint32_t)(127 - X) << 23);
        code = (uint8_t)__nv_cvt_float_to_fp8(__fmul_rn(x, inv), __NV_SATFINITE, __NV_E4M3);
    }
    codes[slot * D + (int64_t)b * 32 + lane] = code;
    if (lane == 0) scales[slot * nb + b] = (uint8_t)E;
}

// Queries rounded onto the MXFP8 grid in one pass: the block exponent and code of
// quantize_mx_kernel, written back as code * 2^(E - 127) in the destination type (the two-kernel
// quantize-then-dequantize result, bit for bit, without the round trip through memory).
template <typename T, typename U>
__global__ void __launch_bounds__(kThreads)
mx_round_kernel(const T* __restrict__ src, int64_t n_rows, int D, U* __restrict__ dst) {
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int nb = D / 32;
    if (warp >= n_rows * nb) return;
    const int64_t i = warp * 32 + lane;            // rows are contiguous: block b of row r
    const float x = to_f32(src[i]);
    float amax = fabsf(x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float v = 0.f;
    if (amax > 0.f) {
        const int X = min(127, max(-127, floor_log2(amax) - 8));
        const float inv = __uint_as_float((uint32_t)(127 - X) << 23);
        const uint8_t code = (uint8_t)__nv_cvt_float_to_fp8(__fmul_rn(x, inv), __NV_SATFINITE, __NV_E4M3);
        v = e4m3_to_f32(code) * e8m0_to_f32((uint32_t)(X + 127));
    }
    if constexpr (sizeof(U) == 4)
        dst[i] = v;
    else
        dst[i] = __float2bfloat16_rn(v);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
dequantize_mx_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                     int64_t n, int D, T* __restrict__ dst) {
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= n) return;
    const int64_t r = i / D;
    const int d = (int)(i % D);
    const float v = e4m3_to_f32(codes[i]) * e8m0_to_f32(scales[r * (D / 32) + d / 32]);
    if constexpr (sizeof(T) == 4)
        dst[i] = v;
    else
        dst[i] = __float2bfloat16_rn(v);
}

}  // namespace

cudaError_t launch_quantize_mx(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D,
                               const int64_t* slot_mapping, int64_t num_slots, uint8_t* codes,
                               uint8_t* scales, cudaStream_t st) {
    if (n_rows == 0) return cudaSuccess;
    const int64_t blocks = ceil_div(n_rows * (D / 32) * 32, kThreads);
    if (src_dtype == HSA_F32)
        quantize_mx_kernel<float><<<(unsigned)blocks, kThreads, 0, st>>>(
            reinterpret_cast<const float*>(src), n_rows, D, slot_mapping, num_slots, codes, scales);
    else
        quantize_mx_kernel<__nv_bfloat16><<<(unsigned)blocks, kThreads, 0, st>>>(
            reinterpret_cast<const __nv_bfloat16*>(src), n_rows, D, slot_mapping, num_slots, codes,
            scales);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_mx_round(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D,
                            void* dst, hsa_dtype_t dst_dtype, cudaStream_t st) {
    if (n_rows == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)ceil_div(n_rows * (D / 32) * 32, kThreads);
    const bool f32_in = src_dtype == HSA_F32, f32_out = dst_dtype == HSA_F32;
    using bf = __nv_bfloat16;
    if (f32_in && f32_out)
        mx_round_kernel<float, float><<<blocks, kThreads, 0, st>>>(
            reinterpret_cast<const float*>(src), n_rows, D, reinterpret_cast<float*>(dst));
    else if (f32_in)
        mx_round_kernel<float, bf><<<blocks, kThreads, 0, st>>>(
            reinterpret_cast<const float*>(src), n_rows, D, reinterpret_cast<bf*>(dst));
    else if (f32_out)
        mx_round_kernel<bf, float><<<blocks, kThreads, 0, st>>>(
            reinterpret_cast<const bf*>(src), n_rows, D, reinterpret_cast<float*>(dst));
    else
        mx_round_kernel<bf, bf><<<blocks, kThreads, 0, st>>>(
            reinterpret_cast<const bf*>(src), n_rows, D, reinterpret_cast<bf*>(dst));
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_dequantize_mx(const uint8_t* codes, const uint8_t* scales, int64_t n_rows,
                                 int32_t D, void* dst, hsa_dtype_t dst_dtype, cudaStream_t st) {
    if (n_rows == 0) return cudaSuccess;
    const int64_t n = n_rows * D;
    const unsigned blocks = (unsigned)ceil_div(n, kThreads);
    if (dst_dtype == HSA_F32)
        dequantize_mx_kernel<float><<<blocks, kThreads, 0, st>>>(codes, scales, n, D,
                                                                 reinterpret_cast<float*>(dst));
    else
        dequantize_mx_kernel<__nv_bfloat16><<<blocks, kThreads, 0, st>>>(
            codes, scales, n, D, reinterpret_cast<__nv_bfloat16*>(dst));
    count_launch();
    return cudaGetLastError();
}

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
