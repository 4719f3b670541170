// common.cuh -- device helpers shared by the libhsa kernels: paged addressing with checks,
// status bits, element loads for the supported storage types.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/hsa.h"

namespace hsa {

// Kernel-side view of hsa_paged_seq_t (copied by value into kernel parameters).
struct SeqView {
    int32_t B;
    const int32_t* seq_lens;
    const int32_t* block_table;
    int64_t bt_stride;
    int32_t page_size;
    int32_t num_pages;
    int32_t max_seq_len;
    int32_t T_q;
    const int32_t* q_seq;
    const int32_t* q_pos;
    uint32_t* status;
};

inline SeqView make_view(const hsa_paged_seq_t& s) {
    SeqView v;
    v.B = s.B;
    v.seq_lens = s.seq_lens;
    v.block_table = s.block_table;
    v.bt_stride = s.bt_stride;
    v.page_size = s.page_size;
    v.num_pages = s.num_pages;
    v.max_seq_len = s.max_seq_len;
    v.T_q = s.T_q;
    v.q_seq = s.q_seq;
    v.q_pos = s.q_pos;
    v.status = s.status;
    return v;
}

__device__ __forceinline__ void flag_status(const SeqView& v, uint32_t bits) {
    if (v.status) atomicOr(v.status, bits);
}

// Validated query row: sequence and position, clamped into range on failure.
struct RowInfo {
    int32_t b;
    int32_t pos;   // -1 when the row is invalid (the row is then skipped)
};

__device__ __forceinline__ RowInfo load_row(const SeqView& v, int32_t t) {
    RowInfo r;
    r.b = __ldg(v.q_seq + t);
    r.pos = __ldg(v.q_pos + t);
    if (r.b < 0 || r.b >= v.B) {
        flag_status(v, HSA_DEV_BAD_POS);
        r.b = 0;
        r.pos = -1;
        return r;
    }
    int32_t len = __ldg(v.seq_lens + r.b);
    if (r.pos < 0 || r.pos >= len || r.pos >= v.max_seq_len) {
        flag_status(v, HSA_DEV_BAD_POS);
        r.pos = -1;
    }
    return r;
}

// Physical slot of logical position s of sequence b.  A page id outside [0, num_pages) is
// reported and redirected to page 0, so the access stays inside the cache.
__device__ __forceinline__ int64_t paged_slot(const SeqView& v, int32_t b, int32_t s) {
    int32_t lp = s / v.page_size;
    int32_t page = __ldg(v.block_table + (int64_t)b * v.bt_stride + lp);
    if (page < 0 || page >= v.num_pages) {
        flag_status(v, HSA_DEV_BAD_PAGE);
        page = 0;
    }
    return (int64_t)page * v.page_size + (s - lp * v.page_size);
}

// The same lookup without a branch on the loaded page: an out-of-range page reads slot 0 of page
// 0 and sets `bad`, which the caller reports once (flag_status) after its loop.  The load's
// result is not needed until the slot is used, so several lookups can be in flight at once.
__device__ __forceinline__ int64_t paged_slot_nb(const SeqView& v, int32_t b, int32_t s, bool& bad) {
    const int32_t lp = s / v.page_size;
    const int32_t page = __ldg(v.block_table + (int64_t)b * v.bt_stride + lp);
    const bool out = (uint32_t)page >= (uint32_t)v.num_pages;
    bad |= out;
    return (int64_t)(out ? 0 : page) * v.page_size + (s - lp * v.page_size);
}

// paged_slot for a page size known to be 2^pshift (pshift >= 0): shifts instead of a division.
__device__ __forceinline__ int64_t paged_slot_pow2(const SeqView& v, int32_t b, int32_t s, int pshift) {
    const int32_t lp = s >> pshift;
    int32_t page = __ldg(v.block_table + (int64_t)b * v.bt_stride + lp);
    if (page < 0 || page >= v.num_pages) {
        flag_status(v, HSA_DEV_BAD_PAGE);
        page = 0;
    }
    return ((int64_t)page << pshift) + (s & ((1 << pshift) - 1));
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// E4M3 code -> float (exact).
__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
    return __half2float(__half(h));
}

// 2^(E - 127) of an E8M0 scale byte (E < 255), exactly: a normal float for E >= 1, the
// subnormal 2^-127 for E = 0.
__device__ __forceinline__ float e8m0_to_f32(uint32_t E) {
    return E ? __uint_as_float(E << 23) : __uint_as_float(1u << 22);
}

template <typename T>
__device__ __forceinline__ float load_f32(const void* p, int64_t i) {
    return to_f32(reinterpret_cast<const T*>(p)[i]);
}

__device__ __forceinline__ float load_any(const void* p, hsa_dtype_t dt, int64_t i) {
    if (dt == HSA_F32) return reinterpret_cast<const float*>(p)[i];
    if (dt == HSA_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
    return e4m3_to_f32(reinterpret_cast<const uint8_t*>(p)[i]);
}

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Kernel launches issued by the calling host thread (reported by hsa_launch_count()).
uint64_t& launch_counter();
inline void count_launch(int n = 1) { launch_counter() += (uint64_t)n; }

// Programmatic dependent launch.  The tensor-core path's kernels (index score, Top-K, sparse MLA)
// are launched so that a kernel may start while the previous kernel on the stream is still
// running.  Such a kernel reads no global memory before pdl_wait() (not even the row
// descriptors: a decode loop may advance q_pos, seq_lens and the block table on the device just
// before the call), which returns once every earlier kernel on the stream has finished and its
// writes are visible; only barrier set-up and the TMEM allocation run before it.  Right after its own
// pdl_wait() it calls pdl_trigger(), which lets the next kernel launch: so when a kernel starts,
// everything before its predecessor has finished.  Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    count_launch();
    return e;
}

}  // namespace hsa
