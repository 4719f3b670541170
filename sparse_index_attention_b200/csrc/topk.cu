// topk.cu -- per-row Top-K by radix select ("Day 0 Inference Adaptation and Optimization for
// Hybrid Attention Models", "Sparse Attention Pipeline Optimization": Top-K of the weighted
// index scores; "Day-One Inference Adaptation for Very Large Hybrid-Attention Models", 3.1).
//
// One 1024-thread CTA per query row.  Scores map to order-preserving 32-bit keys (-0.0 folded
// onto +0.0).  The selection is every key above T, the key of the K-th best element, and the
// lowest-position elements equal to T (ties go to the lower index), written in ascending
// position order.
//
// A histogram over the whole row is expensive here: the scores concentrate in a few exponent
// bins, and the shared-memory atomics on those bins serialize.  So a long row is first cut down
// to candidates:
//   stage     the row's keys go to shared memory (float4 loads), when they fit;
//   sample    4096 evenly spaced keys; a two-pass radix select on them gives a threshold L a few
//             standard deviations below the sample's estimate of T, so that the row holds K or
//             more keys >= L with overwhelming probability;
//   collect   warps sweep contiguous segments of the row and keep every key >= L with its
//             position, in position order: a staged row takes a ballot count, a scan over the
//             warps and a second sweep that writes at the scanned offsets; a row read from L2
//             takes one sweep that appends to a stretch per warp, then the stretches are moved
//             down end to end (the two-sweep form if a stretch overflows);
//   select    a three-pass radix select (digits of 11, 11 and 10 bits) over the candidates finds
//             T exactly and how many elements equal to T are selected;
//   write     a ballot sweep over the candidates places each selected position.
// Whenever the candidates cannot be used -- short rows, too few keys >= L, more than fit in
// shared memory (heavy ties) -- the select and write steps run over the whole row instead, which
// gives the same result.  Either way the output is exact: the threshold only decides how much
// work the exact steps see.
#include <algorithm>

#include "kernels.h"
#include "tc_common.cuh"

namespace hsa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kSample = 4096;
// 32-key groups per warp step of the candidate sweeps: sixteen for rows read from L2 (all
// sixteen reads in flight before the first is used; those sweeps are latency-bound), four for
// rows staged in shared memory (measured faster there)
template <bool kStaged> constexpr int kSweep = kStaged ? 4 : 16;
constexpr int kSampleMinRow = 2 * kSample;     // shorter rows go straight to the exact steps
constexpr int kSmemKeys = 40 * 1024;           // staged keys (160 KB)
constexpr int kMaxSmem = 227 * 1024;
// shared memory ahead of the candidates: histogram, warp sums, scalars
constexpr int kFixedWords = kBins + 2 * kWarps + 16;

__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;              // -0.0 == +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

struct Kth {
    uint32_t key;    // the k-th largest key (with two passes: its top 22 bits, low 10 bits zero)
    uint32_t krem;   // how many elements equal to `key` are among the k largest (three passes)
};

// Radix select over the n keys get(0..n-1) (1 <= k <= n): digits of 11, 11 and 10 bits, most
// significant first; each pass histograms the keys that share the digits found so far.  `hist`
// is all zero on entry and is left all zero: the thread that reads a bin's count clears it.
template <int kPasses, class Get>
__device__ Kth radix_select(const Get& get, int n, uint32_t k, uint32_t* hist, uint64_t* wsum,
                            uint32_t* misc) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t prefix = 0u, pmask = 0u, krem = k;
#pragma unroll 1
    for (int pass = 0; pass < kPasses; ++pass) {
        const int sh = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const uint32_t dmask = pass == 2 ? 0x3FFu : 0x7FFu;
#pragma unroll 1
        for (int i0 = 0; i0 < n; i0 += kThreads) {
            const int i = i0 + tid;
            const bool ok = i < n;
            const uint32_t u = ok ? get(i) : 0u;
            const bool take = ok && (u & pmask) == prefix;
            const uint32_t bin = (u >> sh) & dmask;
            // a warp whose lanes all take one bin (ties, constant rows) adds once
            const uint32_t b0 = __shfl_sync(0xffffffffu, bin, 0);
            if (__all_sync(0xffffffffu, take && bin == b0)) {
                if (lane == 0) atomicAdd(hist + b0, 32u);
            } else if (take) {
                atomicAdd(hist + bin, 1u);
            }
        }
        __syncthreads();
        // thread i owns digits d0 = 2047 - 2i (higher) and d1 = 2046 - 2i: a prefix sum in this
        // order counts the keys whose digit is >= d1
        const int d0 = kBins - 1 - 2 * tid, d1 = d0 - 1;
        const uint32_t h0 = hist[d0], c = h0 + hist[d1];
        hist[d0] = 0u;
        hist[d1] = 0u;
        uint32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        // every warp scans the 32 warp totals itself
        const uint32_t wt = (uint32_t)wsum[lane];
        uint32_t wincl = wt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, wincl, o);
            if (lane >= o) wincl += y;
        }
        const uint32_t wbefore = __shfl_sync(0xffffffffu, wincl - wt, warp);
        const uint32_t excl = wbefore + incl - c;
        if (excl < krem && krem <= excl + c) {
            misc[0] = excl + h0 >= krem ? (uint32_t)d0 : (uint32_t)d1;
            misc[1] = excl + h0 >= krem ? excl : excl + h0;
        }
        __syncthreads();
        krem -= misc[1];
        prefix |= misc[0] << sh;
        pmask |= dmask << sh;
    }
    return Kth{prefix, krem};
}

// Writes the selection -- keys above T, and the first krem keys equal to T -- from the n keys
// get(0..n-1), which are in ascending position order, to out[] in that order.  Warps own
// contiguous segments; a count sweep and a scan over the warps give each its first slot.
template <class Get, class Pos>
__device__ void write_selection(const Get& get, const Pos& pos, int n, uint32_t T, uint32_t krem,
                                int K, int32_t* __restrict__ out, uint64_t* wsum) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int seg = ((n + kThreads - 1) / kThreads) * 32;
    const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
    uint32_t gt = 0u, eq = 0u;
    for (int j = s0; j < s1; j += 32) {
        const int i = j + lane;
        const bool ok = i < s1;
        const uint32_t u = ok ? get(i) : 0u;
        gt += (uint32_t)__popc(__ballot_sync(0xffffffffu, ok && u > T));
        eq += (uint32_t)__popc(__ballot_sync(0xffffffffu, ok && u == T));
    }
    if (lane == 0) wsum[warp] = ((uint64_t)gt << 32) | eq;
    __syncthreads();
    uint64_t before = lane < warp ? wsum[lane] : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
    uint32_t gb = (uint32_t)(before >> 32), eb = (uint32_t)before;
    for (int j = s0; j < s1; j += 32) {
        const int i = j + lane;
        const bool ok = i < s1;
        const uint32_t u = ok ? get(i) : 0u;
        const uint32_t bg = __ballot_sync(0xffffffffu, ok && u > T);
        const uint32_t be = __ballot_sync(0xffffffffu, ok && u == T);
        const uint32_t g = gb + (uint32_t)__popc(bg & lanemask_lt());
        const uint32_t e = eb + (uint32_t)__popc(be & lanemask_lt());
        // the output slot of a selected element is the number of selected elements at lower
        // positions (< K by construction; the bound keeps a wrong count harmless)
        if (ok && u > T) {
            const uint32_t o = g + min(e, krem);
            if (o < (uint32_t)K) out[o] = pos(i);
        } else if (ok && u == T && e < krem && g + e < (uint32_t)K) {
            out[g + e] = pos(i);
        }
        gb += (uint32_t)__popc(bg);
        eb += (uint32_t)__popc(be);
    }
}

template <bool kStaged>
__global__ void __launch_bounds__(kThreads, 1)
topk_kernel(SeqView v, const float* __restrict__ scores, int64_t ld, int K, int cand_cap,
            int32_t* __restrict__ idx) {
    extern __shared__ __align__(16) uint32_t sm[];
    uint32_t* hist = sm;                                          // [kBins]
    uint64_t* wsum = reinterpret_cast<uint64_t*>(sm + kBins);     // [kWarps]
    uint32_t* misc = sm + kBins + 2 * kWarps;                     // [16]
    uint32_t* cand_key = misc + 16;                               // [cand_cap]; first the sample
    uint32_t* cand_pos = cand_key + cand_cap;                     // [cand_cap]
    uint32_t* keys_raw = cand_pos + cand_cap;                     // [n + 4] when staged
    uint32_t* keys = keys_raw;           // staged keys: key i of the row at keys[i]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = blockIdx.x;
    pdl_wait();                          // scores and row descriptors may be earlier kernels' output
    pdl_trigger();
    const RowInfo r = load_row(v, t);
    int32_t* out = idx + (int64_t)t * K;
    const int n = r.pos + 1;             // 0 for an invalid row: all -1
    if (n <= K) {
        for (int i = tid; i < K; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }
    const float* src = scores + (int64_t)t * ld;
    for (int b = tid; b < kBins; b += kThreads) hist[b] = 0u;
    auto key_at = [&](int i) -> uint32_t { return kStaged ? keys[i] : score_key(__ldg(src + i)); };

    if (kStaged) {
        // the row's 16-byte-aligned body arrives by one bulk copy (the copy engine streams a
        // contiguous row much faster than per-thread loads from L2), the unaligned tail by plain
        // loads; then every thread turns its share of the scores into keys in place.  The copy
        // starts at the 16-byte boundary at or below the row (up to three floats of the previous
        // row, never before the allocation, which is at least 16-byte aligned) and ends at or
        // below the row's end.
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(src) & ~uintptr_t(15);
        const uintptr_t a1 = reinterpret_cast<uintptr_t>(src + n) & ~uintptr_t(15);
        const int head = (int)((reinterpret_cast<uintptr_t>(src) - a0) >> 2);   // 0..3 floats
        keys = keys_raw + head;          // element i of the row lands at keys[i]
        uint64_t* bar = reinterpret_cast<uint64_t*>(misc + 10);
        volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 12);
        const uint32_t bytes = (uint32_t)(a1 - a0);
        if (tid == 0) {
            *abort_flag = 0;
            tc::mbar_init(bar, 1);
            tc::fence_barrier_init();
        }
        __syncthreads();
        if (tid == 0) {
            if (bytes > 0) {
                tc::mbar_arrive_expect_tx(bar, bytes);
                tc::bulk_load(keys_raw, reinterpret_cast<const void*>(a0), bytes, bar);
            } else {
                tc::mbar_arrive(bar);
            }
        }
        const int body = max(0, (int)(bytes >> 2) - head);   // row elements the copy covers
        for (int i = body + tid; i < n; i += kThreads) keys[i] = __float_as_uint(__ldg(src + i));
        const bool landed = tc::mbar_wait(bar, 0, abort_flag);
        if (!__syncthreads_and(landed)) {   // the copy never completed: report, skip the row
            if (tid == 0) flag_status(v, HSA_DEV_TIMEOUT);
            return;
        }
        for (int i = tid; i < n; i += kThreads) keys[i] = score_key(__uint_as_float(keys[i]));
    }
    __syncthreads();

    // candidates: the keys >= a threshold taken from a sample, in position order
    int n_cand = -1;                     // -1: the exact steps run over the whole row
    if (n >= kSampleMinRow) {
        const float ps = (float)K * (float)kSample / (float)n;   // expected sample keys >= T
        const int rank = (int)ceilf(ps + 4.f * sqrtf(ps) + 8.f);
        if (rank < kSample / 2) {
            uint32_t* sample = cand_key;
            for (int s = tid; s < kSample; s += kThreads)
                sample[s] = key_at((int)(((int64_t)s * n) / kSample));
            __syncthreads();
            const uint32_t L = radix_select<2>([&](int i) { return sample[i]; }, kSample,
                                               (uint32_t)rank, hist, wsum, misc).key;
            // warp segments of whole 128-key chunks, swept kSweep keys per lane at a time
            const int seg = ((n + kWarps * 128 - 1) / (kWarps * 128)) * 128;
            const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
            // Rows read from L2: one sweep both counts and collects.  Each warp appends its keys
            // >= L, in position order, to its own stretch of the upper half of the candidate
            // arrays (a key past the end of the stretch is counted, not stored), and the
            // stretches are then moved down end to end.  If a stretch overflowed (heavy ties),
            // the second sweep below collects instead.  Staged rows count, then collect.
            constexpr bool kOneSweep = !kStaged;
            const int cap_w = kOneSweep ? (cand_cap / 2) / kWarps : 0;
            uint32_t* own_key = cand_key + cand_cap / 2 + warp * cap_w;
            uint32_t* own_pos = cand_pos + cand_cap / 2 + warp * cap_w;
            const uint32_t lt = lanemask_lt();
            uint32_t c = 0u;
            for (int j = s0; j < s1; j += 32 * kSweep<kStaged>) {
                uint32_t u[kSweep<kStaged>];
#pragma unroll
                for (int a = 0; a < kSweep<kStaged>; ++a) {
                    const int i = j + 32 * a + lane;
                    u[a] = i < s1 ? key_at(i) : 0u;
                }
#pragma unroll
                for (int a = 0; a < kSweep<kStaged>; ++a) {
                    const int i = j + 32 * a + lane;
                    const uint32_t bal = __ballot_sync(0xffffffffu, i < s1 && u[a] >= L);
                    if constexpr (kOneSweep) {
                        const uint32_t p = c + (uint32_t)__popc(bal & lt);
                        if (((bal >> lane) & 1u) && p < (uint32_t)cap_w) {
                            own_key[p] = u[a];
                            own_pos[p] = (uint32_t)i;
                        }
                    }
                    c += (uint32_t)__popc(bal);
                }
            }
            if (lane == 0) wsum[warp] = c;
            const bool spilled = __syncthreads_or(kOneSweep && c > (uint32_t)cap_w);
            uint32_t before = lane < warp ? (uint32_t)wsum[lane] : 0u;
            uint32_t total = (uint32_t)wsum[lane];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                before += __shfl_xor_sync(0xffffffffu, before, o);
                total += __shfl_xor_sync(0xffffffffu, total, o);
            }
            __syncthreads();
            // (every condition below is the same in every thread)
            if (kOneSweep && !spilled && total >= (uint32_t)K && total <= (uint32_t)(cand_cap / 2)) {
                for (uint32_t k = lane; k < c; k += 32) {   // stretch -> [before, before + c)
                    cand_key[before + k] = own_key[k];
                    cand_pos[before + k] = own_pos[k];
                }
                n_cand = (int)total;
                __syncthreads();
            } else if (total >= (uint32_t)K && total <= (uint32_t)cand_cap) {
                for (int j = s0; j < s1; j += 32 * kSweep<kStaged>) {
                    uint32_t u[kSweep<kStaged>], bal[kSweep<kStaged>];
#pragma unroll
                    for (int a = 0; a < kSweep<kStaged>; ++a) {
                        const int i = j + 32 * a + lane;
                        u[a] = i < s1 ? key_at(i) : 0u;
                    }
#pragma unroll
                    for (int a = 0; a < kSweep<kStaged>; ++a) {
                        const int i = j + 32 * a + lane;
                        bal[a] = __ballot_sync(0xffffffffu, i < s1 && u[a] >= L);
                    }
#pragma unroll
                    for (int a = 0; a < kSweep<kStaged>; ++a) {
                        if ((bal[a] >> lane) & 1u) {
                            const uint32_t p = before + (uint32_t)__popc(bal[a] & lt);
                            cand_key[p] = u[a];
                            cand_pos[p] = (uint32_t)(j + 32 * a + lane);
                        }
                        before += (uint32_t)__popc(bal[a]);
                    }
                }
                n_cand = (int)total;
                __syncthreads();
            }
        }
    }

    if (n_cand >= 0) {
        auto get = [&](int i) { return cand_key[i]; };
        const Kth kth = radix_select<3>(get, n_cand, (uint32_t)K, hist, wsum, misc);
        write_selection(get, [&](int i) { return (int32_t)cand_pos[i]; }, n_cand, kth.key, kth.krem,
                        K, out, wsum);
    } else {
        const Kth kth = radix_select<3>(key_at, n, (uint32_t)K, hist, wsum, misc);
        write_selection(key_at, [](int i) { return (int32_t)i; }, n, kth.key, kth.krem, K, out, wsum);
    }
}

template <bool kStaged>
cudaError_t launch_variant(const SeqView& seq, const float* scores, int64_t ld, int32_t K,
                           int cand_cap, size_t smem, int32_t* idx, cudaStream_t st) {
    auto k = topk_kernel<kStaged>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(k, dim3(seq.T_q), dim3(kThreads), smem, st, seq, scores, ld, (int)K, cand_cap, idx);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Block-aligned selection ("Day-One Inference Adaptation for Very Large Hybrid-Attention
// Models", 3.1: the selection is aligned to cache blocks so that the attention reads the cache in
// contiguous pieces).  A row with n > K causal positions keeps the K / block blocks of `block`
// positions with the highest block maximum (ties to the lower block; the last block may be
// partial) and every causal position of each kept block, in ascending order.  One CTA per row:
// the block maxima become keys in shared memory, the radix select above picks the blocks
// exactly, write_selection lists them in block order, and the threads expand them to positions.
__global__ void __launch_bounds__(kThreads, 1)
topk_blocks_kernel(SeqView v, const float* __restrict__ scores, int64_t ld, int K, int block,
                   int32_t* __restrict__ idx) {
    extern __shared__ __align__(16) uint32_t sm[];
    uint32_t* hist = sm;                                          // [kBins]
    uint64_t* wsum = reinterpret_cast<uint64_t*>(sm + kBins);     // [kWarps]
    uint32_t* misc = sm + kBins + 2 * kWarps;                     // [16]
    int32_t* chosen = reinterpret_cast<int32_t*>(misc + 16);      // [K / block] kept blocks
    uint32_t* bkey = misc + 16 + K / block;                       // [blocks of the row]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = blockIdx.x;
    pdl_wait();
    pdl_trigger();
    const RowInfo r = load_row(v, t);
    int32_t* out = idx + (int64_t)t * K;
    const int n = r.pos + 1;
    if (n <= K) {
        for (int i = tid; i < K; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }
    const float* src = scores + (int64_t)t * ld;
    const int nb = (n + block - 1) / block, kb = K / block;
    for (int b = warp; b < nb; b += kWarps) {
        float m = -INFINITY;
        const int s1 = min(n, (b + 1) * block);
        for (int s = b * block + lane; s < s1; s += 32) m = fmaxf(m, __ldg(src + s));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) bkey[b] = score_key(m);
    }
    for (int b = tid; b < kBins; b += kThreads) hist[b] = 0u;
    __syncthreads();
    auto get = [&](int i) { return bkey[i]; };
    const Kth kth = radix_select<3>(get, nb, (uint32_t)kb, hist, wsum, misc);
    write_selection(get, [](int i) { return (int32_t)i; }, nb, kth.key, kth.krem, kb, chosen, wsum);
    __syncthreads();
    // kept block j (ascending) fills slots [j * block, (j + 1) * block); only the last block of
    // the row can be partial, and it is the last kept one if kept, so its missing positions are
    // the -1 padding at the end
    for (int i = tid; i < K; i += kThreads) {
        const int s = chosen[i / block] * block + i % block;
        out[i] = s < n ? s : -1;
    }
}

}  // namespace

cudaError_t launch_topk_blocks(const SeqView& seq, int32_t max_seq_len, const float* scores,
                               int64_t ld, int32_t K, int32_t block, int32_t* idx, cudaStream_t st) {
    if (seq.T_q == 0) return cudaSuccess;
    const size_t smem = sizeof(uint32_t) * ((size_t)kFixedWords + (size_t)(K / block) +
                                            (size_t)ceil_div(max_seq_len, block));
    auto k = topk_blocks_kernel;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(k, dim3(seq.T_q), dim3(kThreads), smem, st, seq, scores, ld, (int)K, (int)block, idx);
    return e != cudaSuccess ? e : cudaGetLastError();
}

size_t topk_blocks_smem(int32_t max_seq_len, int32_t K, int32_t block) {
    return sizeof(uint32_t) * ((size_t)kFixedWords + (size_t)(K / block) + (size_t)ceil_div(max_seq_len, block));
}

cudaError_t launch_topk(const SeqView& seq, int32_t max_seq_len, const float* scores, int64_t ld,
                        int32_t K, int32_t* idx, cudaStream_t st) {
    if (seq.T_q == 0) return cudaSuccess;
    const bool staged = max_seq_len <= kSmemKeys;
    const int staged_words = staged ? ((max_seq_len + 3) & ~3) + 4 : 0;   // + up to 3 floats of head
    // candidates (key and position) fill the rest; always room for the sample
    const int cand_cap = ((kMaxSmem / 4 - kFixedWords - staged_words) / 2) & ~3;
    const size_t smem = sizeof(uint32_t) * ((size_t)kFixedWords + 2 * (size_t)cand_cap + staged_words);
    static_assert((kMaxSmem / 4 - kFixedWords - kSmemKeys) / 2 >= kSample, "no room for the sample");
    return staged ? launch_variant<true>(seq, scores, ld, K, cand_cap, smem, idx, st)
                  : launch_variant<false>(seq, scores, ld, K, cand_cap, smem, idx, st);
}

}  // namespace hsa
