// topk.cu -- per-row Top-K by radix select ("Day 0 Inference Adaptation and Optimization for
// Hybrid Attention Models", "Sparse Attention Pipeline Optimization": Top-K of the weighted
// index scores; "Day-One Inference Adaptation for Very Large Hybrid-Attention Models", 3.1).
//
// One 1024-thread CTA per query row.  Scores map to order-preserving 32-bit keys (-0.0 folded
// onto +0.0).  Three histogram passes over digits of 11, 11 and 10 bits find the exact key T
// of the K-th best element and how many elements equal to T belong to the selection.  A final
// pass compacts the selection in ascending position order with a block-wide scan: every key
// above T, and the lowest-position elements equal to T (ties go to the lower index).  Rows of
// at most kSmemKeys positions are staged once in shared memory; longer rows are re-read from
// global memory (L2) on every pass.
#include "kernels.h"

namespace hsa {

namespace {

constexpr int kThreads = 1024;
constexpr int kBins = 2048;
constexpr int kItems = 16;                     // consecutive positions per thread in compaction
constexpr int kSmemKeys = 50 * 1024;           // 200 KB of staged keys

__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;              // -0.0 == +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive scan of one value per thread over the whole block; `total` gets the block sum.
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t x, uint32_t* wsum, uint32_t& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kWarps = kThreads / 32;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = lane < kWarps ? wsum[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        wsum[lane] = s;
    }
    __syncthreads();
    const uint32_t pre = warp > 0 ? wsum[warp - 1] : 0u;
    total = wsum[kWarps - 1];
    __syncthreads();
    return x + pre;
}

template <bool kStaged>
__global__ void __launch_bounds__(kThreads, 1)
topk_kernel(SeqView v, const float* __restrict__ scores, int64_t ld, int K, int32_t* __restrict__ idx) {
    extern __shared__ uint32_t sm[];
    uint32_t* hist = sm;                 // [kBins]
    uint32_t* wsum = sm + kBins;         // [32]
    uint32_t* misc = wsum + 32;          // [8]
    uint32_t* keys = misc + 8;           // [n] when staged
    const int t = blockIdx.x;
    const RowInfo r = load_row(v, t);
    int32_t* out = idx + (int64_t)t * K;
    const int n = r.pos + 1;             // 0 for an invalid row: all -1
    if (n <= K) {
        for (int i = threadIdx.x; i < K; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }
    const float* row = scores + (int64_t)t * ld;
    if (kStaged) {
        for (int i = threadIdx.x; i < n; i += kThreads) keys[i] = score_key(row[i]);
        __syncthreads();
    }
    auto key_at = [&](int i) -> uint32_t { return kStaged ? keys[i] : score_key(__ldg(row + i)); };

    uint32_t prefix = 0u, pmask = 0u, krem = (uint32_t)K;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int sh = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const uint32_t dmask = pass == 2 ? 0x3FFu : 0x7FFu;
        for (int b = threadIdx.x; b < kBins; b += kThreads) hist[b] = 0u;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += kThreads) {
            const uint32_t u = key_at(i);
            if ((u & pmask) == prefix) atomicAdd(&hist[(u >> sh) & dmask], 1u);
        }
        __syncthreads();
        // thread i owns digits d0 = 2047 - 2i (higher) and d1 = 2046 - 2i: a prefix scan in this
        // order counts the elements whose digit is >= d1
        const int d0 = kBins - 1 - 2 * threadIdx.x, d1 = d0 - 1;
        const uint32_t h0 = hist[d0], c = h0 + hist[d1];
        uint32_t total;
        const uint32_t incl = block_incl_scan(c, wsum, total);
        const uint32_t excl = incl - c;
        if (excl < krem && krem <= incl) {
            if (excl + h0 >= krem) {
                misc[0] = (uint32_t)d0;
                misc[1] = excl;
            } else {
                misc[0] = (uint32_t)d1;
                misc[1] = excl + h0;
            }
        }
        __syncthreads();
        const uint32_t digit = misc[0], above = misc[1];
        krem -= above;
        prefix |= digit << sh;
        pmask |= dmask << sh;
        __syncthreads();
    }
    // prefix is the exact key T of the K-th best element; krem (>= 1) elements equal to T are
    // selected, the ones at the lowest positions.
    const uint32_t T = prefix;
    uint32_t run_gt = 0u, run_eq = 0u;
#pragma unroll 1
    for (int base = 0; base < n; base += kThreads * kItems) {
        const int p0 = base + threadIdx.x * kItems;
        uint32_t u[kItems];
        uint32_t gt = 0u, eq = 0u;
#pragma unroll
        for (int k = 0; k < kItems; ++k) {
            u[k] = (p0 + k < n) ? key_at(p0 + k) : 0u;
            gt += (p0 + k < n) && u[k] > T;
            eq += (p0 + k < n) && u[k] == T;
        }
        // both counts fit in 16 bits (at most kThreads * kItems = 16384 per chunk)
        uint32_t total;
        const uint32_t incl = block_incl_scan((gt << 16) | eq, wsum, total);
        const uint32_t excl = incl - ((gt << 16) | eq);
        uint32_t gb = run_gt + (excl >> 16), eb = run_eq + (excl & 0xFFFFu);
#pragma unroll
        for (int k = 0; k < kItems; ++k) {
            if (p0 + k >= n) break;
            // the output slot of a selected element is the number of selected elements at
            // lower positions (< K by construction; the bound keeps a wrong count harmless)
            if (u[k] > T) {
                const uint32_t o = gb + min(eb, krem);
                if (o < (uint32_t)K) out[o] = p0 + k;
                ++gb;
            } else if (u[k] == T) {
                if (eb < krem && gb + eb < (uint32_t)K) out[gb + eb] = p0 + k;
                ++eb;
            }
        }
        run_gt += total >> 16;
        run_eq += total & 0xFFFFu;
    }
}

}  // namespace

cudaError_t launch_topk(const SeqView& seq, int32_t max_seq_len, const float* scores, int64_t ld,
                        int32_t K, int32_t* idx, cudaStream_t st) {
    if (seq.T_q == 0) return cudaSuccess;
    const size_t base = sizeof(uint32_t) * (kBins + 32 + 8);
    if (max_seq_len <= kSmemKeys) {
        const size_t smem = base + sizeof(uint32_t) * (size_t)max_seq_len;
        auto k = topk_kernel<true>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k<<<seq.T_q, kThreads, smem, st>>>(seq, scores, ld, K, idx);
    count_launch();
    } else {
        topk_kernel<false><<<seq.T_q, kThreads, base, st>>>(seq, scores, ld, K, idx);
    count_launch();
    }
    return cudaGetLastError();
}

}  // namespace hsa
