// index_score_tc.cu -- tensor-core index score for the 64-head x 128-dim indexer (sm_100a).
//
// I[t,s] = sum_j w[t,j] ReLU(q_I[t,j,:] . k[s,:])  ("Day 0 Inference Adaptation and Optimization
// for Hybrid Attention Models", "Sparse Attention Pipeline Optimization": per-head scores over
// the paged K cache, combined with the per-head weights; fifth page, 3.1).
//
// Mapping.  One tcgen05 MMA tile is D[128 keys x G*64] = K_tile[128 x 128] . Q_group^T, with the
// keys on M (TMEM lanes) and G query rows x 64 index heads on N (TMEM columns).  The epilogue
// thread that owns TMEM lane r owns key s = tile*128 + r and reduces its 64 head columns per
// query row in registers: no cross-thread reduction.  Accumulators are multi-buffered in TMEM
// (four for N <= 128, two for N = 256) so the epilogue of tile i overlaps the MMAs of the next.
//
// Schedule.  Work is the flat list of (query group, key tile) pairs, where a group is G
// consecutive rows of one sequence and its key range is [0, max position of the group].  Each
// persistent CTA takes one contiguous slice of that list (load balance without atomics), so
// it walks the keys of one group in order and reloads the group's queries only when the group
// changes.  Every CTA derives the list itself from q_pos (prefix sum in shared memory).
//
// Data movement.  Keys come through the block table page by page with 2D TMA loads (128-byte
// swizzle, two 64-column halves per page).  E4M3 keys (with a 16-byte-aligned scale array) go
// straight from TMA to 8-bit MMAs (kind::f8f6f4): each bf16 query row x head is split into two
// E4M3 code rows, hi and lo (scaled per head by a power of two folded into its weight), and the
// MMAs of both accumulate into one accumulator, hi . k + lo . k = q . k; the per-key fp32
// scales are bulk-copied beside the codes for the epilogue.  Otherwise the E4M3 codes are
// loaded raw and widened in shared memory by converter warps (E4M3 -> f16 in one conversion,
// exact; the MMA then runs in f16, the queries rescaled into f16's range per head).  Either way
// the per-key fp32 scale multiplies the finished score (the scale is positive, so it commutes
// with the ReLU sum).  MXFP8 keys (one E8M0 byte per 32 dims; "Inference Adaptation and
// Performance Optimization for a Domestically Developed LLM's New Architecture", section 4
// table) with bf16 queries are widened too: the producer bulk-copies each box's scale words
// beside its codes, the converters place the codes' bits in bf16s and scale each 32-dim block
// by 2^(E_block - E_max) with one packed multiply (exact), and the epilogue multiplies the score
// by 2^(E_max - 127), the key's largest block scale.  MXFP8 keys with MXFP8 queries skip the
// converters: the codes go straight to a block-scaled MMA (kind::mxf8f6f4) that reads the E8M0
// scales from TMEM.
//
// Warp roles: 0 TMA producer, 1 MMA issuer (one elected thread each), 2-5 epilogue
// (TMEM lane quarters 2,3,0,1), 6-9 (6-13 for E4M3 keys with one row per tile) FP8 converters
// when the codes are widened, or 6-9 key-scale writers (block-scaled MMA); with two or four
// rows per tile four more epilogue warps after those, each pair of a lane quarter summing half
// of the rows.
#include <algorithm>

#include "kernels.h"
#include "tc_common.cuh"

namespace hsa {

namespace {

constexpr int kBM = 128;                 // keys per tile = MMA M
constexpr int kDI = 128;                 // index dim
constexpr int kHI = 64;                  // index heads
constexpr int kHalfBytes = kBM * 128;    // one 64-column swizzled half of a key tile: 16 KB
constexpr int kTileBytes = 2 * kHalfBytes;

template <int G, bool kFp8, bool kMx = false, bool kBs = false, bool kSp = false>
struct Cfg {
    static_assert(!kBs || (G <= 2 && !kFp8 && !kMx), "block-scaled: codes straight to the MMA, G <= 2");
    static_assert(!kSp || (!kFp8 && !kMx && !kBs), "split queries: E4M3 codes straight to the MMA");
    static constexpr int N = G * kHI;   // MMA N = TMEM columns per accumulator
    static constexpr int kTile = (kBs || kSp) ? kBM * kDI : kTileBytes;  // one MMA stage: 16 KB codes or 32 KB bf16
    static constexpr int kQBytes = N * kDI * (kBs ? 1 : 2);
    static constexpr int kStages = kSp ? (G == 1 ? 12 : (G == 2 ? 10 : 8)) : kBs ? (G == 1 ? 8 : 6)
                                       : kFp8 ? (G == 1 ? 4 : (G == 2 ? 3 : 2)) : (G == 1 ? 6 : (G == 2 ? 5 : 4));
    static constexpr int kRawStages = kFp8 ? 4 : 0;          // FP8 staging tiles (16 KB each)
    static constexpr int kR = kRawStages > 0 ? kRawStages : 1;
    // 4 E8M0 bytes or one fp32 scale per key
    static constexpr int kScaleStageBytes = (kMx || kBs || kSp) ? kBM * 4 : 0;
    static constexpr int kScaleStages = (kBs || kSp) ? kStages : kRawStages;
    static constexpr int kMaxGroups = G == 1 ? 2048 : 4096;
    // TMEM: kAcc accumulators of N columns (four for N <= 128, so the MMA may run up to four
    // tiles ahead of the epilogue; two for N = 256); block-scaled adds the key scales (4 columns
    // per stage) and the query scales (N / 32 columns) after them
    static constexpr int kAcc = (N <= 64 || (N == 128 && !kBs)) ? 4 : 2;
    static constexpr int kSfaCol = kAcc * N;
    static constexpr int kSfbCol = kSfaCol + 4 * kStages;
    static constexpr int kTmemCols = kBs ? 512 : kAcc * N;   // 256 or 512
    static_assert(!kBs || kSfbCol + N / 32 <= kTmemCols, "TMEM budget");
    static_assert(kAcc * N <= kTmemCols, "TMEM budget");
    // FP8 converter warps: eight for E4M3 keys with one query row per tile (the widening sets the
    // pace of the key stream there), four otherwise (measured: the MX widening is slower with eight)
    static constexpr int kConv = kFp8 ? ((G == 1 && !kMx) ? 8 : 4) : 0;
    // epilogue warps: four (one per TMEM lane quarter), or eight with two or four rows per tile
    // (two warps per quarter, each summing half of the rows: there the epilogue sets the pace);
    // the second four come after the converter / key-scale warps
    static constexpr int kEpiWarps = (G >= 2 && !kBs) ? 8 : 4;
    static constexpr int kEpiB0 = 6 + (kFp8 ? kConv : (kBs ? 4 : 0));
    static constexpr int kThreads = 32 * (kEpiB0 + (kEpiWarps == 8 ? 4 : 0));
    static constexpr int kBarBytes = kStages > 10 ? 640 : 512;
    static constexpr size_t kSmem = 1024 + (size_t)kStages * kTile + (size_t)kRawStages * (kBM * kDI) +
                                    (size_t)kScaleStages * kScaleStageBytes + kQBytes +
                                    4 * (kMaxGroups + 1) + 4 * N + kBarBytes;
    static_assert(kSmem <= 232448, "shared memory budget");
};

// floor(log2(a)) of a positive finite float, from its bits (subnormals included).
__device__ __forceinline__ int floor_log2_f(float a) {
    const uint32_t bits = __float_as_uint(a);
    const int e = (int)(bits >> 23);
    if (e) return e - 127;
    return (31 - __clz((int)(bits & 0x7FFFFFu))) - 149;
}

struct GroupInfo {
    int32_t b;        // sequence (of the group's first valid row)
    int32_t pos_max;  // largest valid position in the group, -1 if none
};

__device__ __forceinline__ GroupInfo group_info(const SeqView& v, int g, int G, bool flag) {
    GroupInfo gi{-1, -1};
    for (int j = 0; j < G; ++j) {
        const int t = g * G + j;
        if (t >= v.T_q) break;
        RowInfo r = load_row(v, t);
        if (r.pos < 0) continue;
        if (gi.b < 0) gi.b = r.b;
        if (r.b != gi.b) {
            if (flag) flag_status(v, HSA_DEV_BAD_GROUP);
            continue;
        }
        gi.pos_max = max(gi.pos_max, r.pos);
    }
    return gi;
}

// (group, key tile) of flat tile index f, advancing a monotone cursor.
__device__ __forceinline__ void locate(const int32_t* prefix, int n_groups, int64_t f, int& g, int& kt) {
    while (g + 1 < n_groups && prefix[g + 1] <= f) ++g;
    kt = (int)(f - prefix[g]);
}

__device__ __forceinline__ int first_group(const int32_t* prefix, int n_groups, int64_t f) {
    int lo = 0, hi = n_groups - 1;  // last g with prefix[g] <= f
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= f) lo = mid; else hi = mid - 1;
    }
    return lo;
}

template <int G, bool kFp8, bool kMx, bool kBs = false, bool kSp = false>
__global__ void __launch_bounds__(Cfg<G, kFp8, kMx, kBs, kSp>::kThreads, 1)
index_score_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                      SeqView v, int32_t q_row0, const float* __restrict__ w,
                      const void* __restrict__ k_scale, const uint32_t* __restrict__ q_scale,
                      float* __restrict__ scores, int64_t ld, int32_t box_rows) {
    using C = Cfg<G, kFp8, kMx, kBs, kSp>;
    static_assert(!kMx || kFp8, "MXFP8 keys go through the FP8 staging path");
    // kSp (E4M3 keys with fp32 scales, bf16 queries): the key codes go from TMA straight to
    // kind::f8f6f4 MMAs.  Each bf16 query row x head is split into two E4M3 code rows, hi and lo
    // (below), and both MMAs accumulate into one accumulator: hi . k + lo . k = q . k.
    constexpr bool kKeyScale = kFp8 || kSp;   // a per-key scale multiplies the finished score
    constexpr bool kCodes = kBs || kSp;       // 8-bit codes straight into the MMA stages
    // E4M3 keys with fp32 scales run the MMA in f16: a code widens to f16 in one conversion
    // (exact), and the queries are rescaled per head by a power of two into f16's range, the
    // inverse power folded into the head weight, which leaves every product and sum as in bf16.
    constexpr bool kF16 = kFp8 && !kMx;
    constexpr int N = C::N;
    constexpr int S = C::kStages;
    constexpr uint32_t kIdesc = kSp ? tc::idesc_e4m3_f32(kBM, N)
                              : kF16 ? tc::idesc_f16_f32(kBM, N) : tc::idesc_bf16_f32(kBM, N, 0, 0);
    // kBs (MXFP8 queries and keys): the codes go from TMA straight to a block-scaled MMA
    // (kind::mxf8f6f4, K = 32 per instruction, one E8M0 scale per 32 dims of every key and
    // query row, read from TMEM); warps 6-9 place each tile's key scales in TMEM, the epilogue
    // warps each group's query scales.

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* tiles = base;                                          // S x 32 KB bf16 (16 KB codes), swizzled
    uint8_t* raw = tiles + (size_t)S * C::kTile;                    // FP8 staging
    uint8_t* kscl = raw + (size_t)C::kRawStages * (kBM * kDI);      // MXFP8 scale words [4 or S][128]
    uint8_t* qbuf = kscl + (size_t)C::kScaleStages * C::kScaleStageBytes;  // N x 128 bf16 (codes), swizzled
    // barriers first (8-byte alignment), then the variable-size arrays
    uint64_t* bars = reinterpret_cast<uint64_t*>(qbuf + C::kQBytes);
    uint64_t* full = bars;                 // [S]  keys landed (bf16 tile ready)
    uint64_t* empty = full + S;            // [S]  MMA done with the tile
    uint64_t* acc_full = empty + S;        // [kAcc]
    uint64_t* acc_empty = acc_full + 4;    // [kAcc]
    uint64_t* q_full = acc_empty + 4;
    uint64_t* q_empty = q_full + 1;
    uint64_t* raw_full = q_empty + 1;      // [kR] FP8 bytes landed
    uint64_t* raw_empty = raw_full + 8;    // [kR] converters done with the staging tile
    uint64_t* epi_bar = raw_empty + 8;     // the four epilogue warps
    uint64_t* q_ready = epi_bar + 1;       // f16 MMA: the group's queries converted; block-scaled:
                                           // the group's query scales in TMEM (4 warps)
    uint64_t* sf_full = q_ready + 1;       // [S] block-scaled: the tile's key scales in TMEM (4 warps);
                                           // split queries: the epilogue is done with them (4 warps)
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sf_full + S);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    static_assert((3 * S + 4 + 4 + 2 + 16 + 2) * 8 + 8 <= C::kBarBytes && C::kR <= 8 && C::kAcc <= 4, "barrier block");
    int32_t* prefix = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(bars) + C::kBarBytes);
    float* w_s = reinterpret_cast<float*>(prefix + C::kMaxGroups + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_groups = (int)ceil_div(v.T_q, G);

    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            tc::mbar_init(&full[i], kFp8 ? 32 * C::kConv : 1);
            tc::mbar_init(&empty[i], 1);
            tc::mbar_init(&sf_full[i], kSp ? C::kEpiWarps : 4);
        }
        for (int i = 0; i < C::kAcc; ++i) {
            tc::mbar_init(&acc_full[i], 1);
            tc::mbar_init(&acc_empty[i], C::kEpiWarps);
        }
        tc::mbar_init(q_full, 1);
        tc::mbar_init(q_empty, 1);
        for (int i = 0; i < C::kR; ++i) {
            tc::mbar_init(&raw_full[i], 1);
            tc::mbar_init(&raw_empty[i], 32 * C::kConv);
        }
        tc::mbar_init(epi_bar, C::kEpiWarps);
        tc::mbar_init(q_ready, C::kEpiWarps);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_holder, C::kTmemCols);
        tc::tmem_relinquish();
    }
    // the row descriptors and the queries, weights and keys may all be written by the previous
    // kernel on the stream (a decode loop advances q_pos and seq_lens on the device), so nothing
    // of them is read before this wait
    pdl_wait();
    pdl_trigger();
    // tiles per group, then an exclusive prefix sum (warp 0)
    for (int g = tid; g < n_groups; g += blockDim.x) {
        const GroupInfo gi = group_info(v, g, G, blockIdx.x == 0);
        prefix[g] = gi.pos_max >= 0 ? (int32_t)ceil_div(gi.pos_max + 1, kBM) : 0;
    }
    __syncthreads();
    if (warp == 0) {
        int32_t carry = 0;
        for (int g0 = 0; g0 < n_groups; g0 += 32) {
            const int g = g0 + lane;
            int32_t x = g < n_groups ? prefix[g] : 0;
            int32_t incl = x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (g < n_groups) prefix[g] = carry + incl - x;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) prefix[n_groups] = carry;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int64_t total = n_groups > 0 ? prefix[n_groups] : 0;
    const int64_t f_begin = total * blockIdx.x / gridDim.x;
    const int64_t f_end = total * (blockIdx.x + 1) / gridDim.x;

    if (f_begin < f_end) {
        if (warp == 0) {
            // ------------------------------------------------------------ TMA producer
            if (tc::elect_one()) {
                tc::tma_prefetch_desc(&tmap_k);
                tc::tma_prefetch_desc(&tmap_q);
                int g = first_group(prefix, n_groups, f_begin), kt, cur = -1;
                uint32_t stage = 0, phase = 0, qe_phase = 0;
                GroupInfo gi{0, -1};
                // box_rows is a power of two (the page size, 8..128, or 128); so usually is the page
                // size: shifts keep this one thread's per-tile work short
                const int box_shift = __ffs(box_rows) - 1;
                const int pshift = (v.page_size & (v.page_size - 1)) == 0 ? __ffs(v.page_size) - 1 : -1;
                for (int64_t f = f_begin; f < f_end; ++f) {
                    locate(prefix, n_groups, f, g, kt);
                    if (g != cur) {
                        if (cur >= 0) {
                            if (!tc::mbar_wait(q_empty, qe_phase, abort_flag)) break;
                            qe_phase ^= 1;
                        }
                        tc::mbar_arrive_expect_tx(q_full, C::kQBytes);
                        const int32_t qrow = q_row0 + g * G * kHI;
                        tc::tma_load_2d(qbuf, &tmap_q, q_full, 0, qrow);
                        if (!kBs) tc::tma_load_2d(qbuf + N * 128, &tmap_q, q_full, 64, qrow);
                        gi = group_info(v, g, G, false);
                        cur = g;
                    }
                    const int s0 = kt * kBM;
                    const int n_keys = min(kBM, gi.pos_max + 1 - s0);
                    const int n_boxes = (n_keys + box_rows - 1) >> box_shift;
                    uint64_t* bar = kFp8 ? &raw_full[stage % C::kR] : &full[stage];
                    if (kFp8) {
                        if (!tc::mbar_wait(&raw_empty[stage % C::kR], ((stage / C::kR) & 1) ^ 1, abort_flag)) break;
                    } else {
                        if (!tc::mbar_wait(&empty[stage], phase ^ 1, abort_flag)) break;
                        // the stage's key scales outlive the MMA: the epilogue reads them
                        if (kSp && !tc::mbar_wait(&sf_full[stage], phase ^ 1, abort_flag)) break;
                    }
                    tc::mbar_arrive_expect_tx(
                        bar, (uint32_t)(n_boxes * box_rows * (kFp8 ? (kMx ? 132 : 128) : kCodes ? 132 : 256)));
                    for (int j = 0; j < n_boxes; ++j) {
                        const int s = s0 + j * box_rows;
                        const int32_t row = (int32_t)(pshift >= 0 ? paged_slot_pow2(v, gi.b, s, pshift)
                                                                  : paged_slot(v, gi.b, s));
                        if (kFp8) {
                            uint8_t* dst = raw + (size_t)(stage % C::kR) * (kBM * kDI) + (size_t)j * box_rows * 128;
                            tc::tma_load_2d(dst, &tmap_k, bar, 0, row);
                            if (kMx)   // the box's E8M0 words: box_rows x 4 bytes, 32-byte aligned
                                tc::bulk_load(kscl + (size_t)(stage % C::kR) * C::kScaleStageBytes + (size_t)j * box_rows * 4,
                                              static_cast<const uint8_t*>(k_scale) + (int64_t)row * 4,
                                              (uint32_t)box_rows * 4, bar);
                        } else if (kCodes) {   // codes straight into the MMA stage, scales beside
                            // (E8M0 words or fp32, 4 bytes per key; row is a multiple of box_rows,
                            // so the copy is 32-byte aligned and ends inside the scale array)
                            uint8_t* dst = tiles + (size_t)stage * C::kTile + (size_t)j * box_rows * 128;
                            tc::tma_load_2d(dst, &tmap_k, bar, 0, row);
                            tc::bulk_load(kscl + (size_t)stage * C::kScaleStageBytes + (size_t)j * box_rows * 4,
                                          static_cast<const uint8_t*>(k_scale) + (int64_t)row * 4,
                                          (uint32_t)box_rows * 4, bar);
                        } else {
                            uint8_t* dst = tiles + (size_t)stage * kTileBytes + (size_t)j * box_rows * 128;
                            tc::tma_load_2d(dst, &tmap_k, bar, 0, row);
                            tc::tma_load_2d(dst + kHalfBytes, &tmap_k, bar, 64, row);
                        }
                    }
                    if (kFp8) {
                        ++stage;   // staging ring of kR; the MMA ring is advanced by the converters
                    } else if (++stage == (uint32_t)S) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            __syncwarp();
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA issuer
            if (tc::elect_one()) {
                int g = first_group(prefix, n_groups, f_begin), kt, cur = -1;
                uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0, q_phase = 0;
                const uint32_t q_addr = tc::smem_u32(qbuf);
                for (int64_t f = f_begin; f < f_end; ++f) {
                    locate(prefix, n_groups, f, g, kt);
                    if (g != cur) {
                        if (!tc::mbar_wait((kF16 || kSp) ? q_ready : q_full, q_phase, abort_flag)) break;
                        if (kBs && !tc::mbar_wait(q_ready, q_phase, abort_flag)) break;
                        q_phase ^= 1;
                        cur = g;
                    }
                    if (!tc::mbar_wait(&full[stage], phase, abort_flag)) break;
                    if (kBs && !tc::mbar_wait(&sf_full[stage], phase, abort_flag)) break;
                    if (!tc::mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag)) break;
                    tc::tc_fence_after();
                    const uint32_t a_addr = tc::smem_u32(tiles + (size_t)stage * C::kTile);
                    const uint32_t d = tmem_base + acc * N;
                    if (kSp) {
                        // four K = 32 steps through the 128-byte code rows of the keys against the
                        // hi query rows, then four against the lo rows (N rows further on), all
                        // into the one accumulator
#pragma unroll
                        for (int k = 0; k < 2 * (kDI / 32); ++k)
                            tc::mma_f8(d, tc::sw128_desc(a_addr + (k & 3) * 32, 16, 1024),
                                       tc::sw128_desc(q_addr + (k >> 2) * (N * 128) + (k & 3) * 32, 16, 1024),
                                       kIdesc, k > 0 ? 1u : 0u);
                    } else if (kBs) {
                        // four K = 32 steps through the 128-byte code rows; step k reads byte k
                        // of every key's and query row's scale word
#pragma unroll
                        for (int k = 0; k < kDI / 32; ++k) {
                            const uint32_t sel = (uint32_t)k << 30;
                            tc::mma_mxf8(d, tc::sw128_desc(a_addr + k * 32, 16, 1024),
                                         tc::sw128_desc(q_addr + k * 32, 16, 1024),
                                         tc::idesc_mxf8_f32(kBM, N, k, k),
                                         (tmem_base + C::kSfaCol + 4 * stage) | sel,
                                         (tmem_base + C::kSfbCol) | sel, k > 0 ? 1u : 0u);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < kDI / 16; ++k) {
                            const uint32_t koff = (uint32_t)((k >> 2) * kHalfBytes + (k & 3) * 32);
                            const uint32_t qoff = (uint32_t)((k >> 2) * (N * 128) + (k & 3) * 32);
                            tc::mma_bf16(d, tc::sw128_desc(a_addr + koff, 16, 1024),
                                         tc::sw128_desc(q_addr + qoff, 16, 1024), kIdesc, k > 0 ? 1u : 0u);
                        }
                    }
                    tc::mma_commit(&empty[stage]);
                    tc::mma_commit(&acc_full[acc]);
                    int g2 = g, kt2;
                    if (f + 1 < f_end) locate(prefix, n_groups, f + 1, g2, kt2);
                    if (f + 1 == f_end || g2 != g) tc::mma_commit(q_empty);
                    if (++stage == (uint32_t)S) {
                        stage = 0;
                        phase ^= 1;
                    }
                    if (++acc == (uint32_t)C::kAcc) {
                        acc = 0;
                        acc_phase ^= 1;
                    }
                }
            }
            __syncwarp();
        } else if (warp < 6 || (C::kEpiWarps == 8 && warp >= C::kEpiB0)) {
            // ------------------------------------------------------------ epilogue
            const int quarter = warp & 3;
            const int r_in_tile = quarter * 32 + lane;
            constexpr int kEpiThreads = 32 * C::kEpiWarps;
            const int ehalf = warp >= 6 ? 1 : 0;      // second epilogue warp of its lane quarter
            const int et = ehalf ? 128 + tid - 32 * C::kEpiB0 : tid - 64;   // 0 .. kEpiThreads - 1
            // the row groups this warp sums: all, or its half of them
            const int jlo = C::kEpiWarps == 8 ? ehalf * (G / 2) : 0;
            const int jhi = C::kEpiWarps == 8 ? jlo + G / 2 : G;
            int g = first_group(prefix, n_groups, f_begin), kt, cur = -1;
            uint32_t acc = 0, acc_phase = 0;
            int32_t row_pos[G];
            int32_t seq_b = 0;
            const int epi_pshift = (v.page_size & (v.page_size - 1)) == 0 ? __ffs(v.page_size) - 1 : -1;
            uint32_t qf_phase = 0;
            uint32_t es = 0, ephase = 0;   // split queries: the key-scale slot of tile f
            tc::WarpSetSync epi_sync{epi_bar, 0};
            for (int64_t f = f_begin; f < f_end; ++f) {
                locate(prefix, n_groups, f, g, kt);
                if (g != cur) {
                    if (!epi_sync.sync(abort_flag)) break;   // everyone is done with the old weights
                    if (kF16) {
                        // the group's queries (TMA-landed bf16, two 64-dim swizzled halves) become
                        // f16 in place: row i (query row x head) is scaled by 2^-e so that its
                        // largest magnitude lies in [2^14, 2^15), and its weight by 2^e; two
                        // threads per row, one per half
                        if (!tc::mbar_wait(q_full, qf_phase, abort_flag)) break;
                        qf_phase ^= 1;
                        const int hf = et & 1;
                        for (int i = et >> 1; i < N; i += kEpiThreads / 2) {
                            uint4* rowp = reinterpret_cast<uint4*>(qbuf + (size_t)hf * (N * 128) + (size_t)i * 128);
                            uint4 x[8];
                            float mx = 0.f;
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                x[c] = rowp[c];
                                const uint32_t wv[4] = {x[c].x, x[c].y, x[c].z, x[c].w};
#pragma unroll
                                for (int qq = 0; qq < 4; ++qq) {
                                    const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[qq]));
                                    mx = fmaxf(mx, fmaxf(fabsf(f2.x), fabsf(f2.y)));
                                }
                            }
                            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                            const int e = mx > 0.f ? min(100, max(-100, floor_log2_f(mx) - 14)) : 0;
                            const float f = __uint_as_float((uint32_t)(127 - e) << 23);
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                uint32_t wv[4] = {x[c].x, x[c].y, x[c].z, x[c].w};
#pragma unroll
                                for (int qq = 0; qq < 4; ++qq) {
                                    const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[qq]));
                                    const __half2 h2 = __floats2half2_rn(f2.x * f, f2.y * f);
                                    wv[qq] = *reinterpret_cast<const uint32_t*>(&h2);
                                }
                                rowp[c] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                            }
                            if (hf == 0) {
                                const int t = g * G + i / kHI;
                                w_s[i] = t < v.T_q ? w[(int64_t)t * kHI + (i % kHI)] *
                                                         __uint_as_float((uint32_t)(127 + e) << 23)
                                                   : 0.f;
                            }
                        }
                        tc::fence_async_smem();   // the f16 queries -> the tensor core
                    } else if (kSp) {
                        // the group's queries (TMA-landed bf16, two 64-dim swizzled halves) become
                        // E4M3 code rows in place.  Row i (query row x head) is scaled by 2^-e so
                        // that its largest magnitude x_max lies in [2^7, 2^8), its weight by 2^e;
                        // then hi = E4M3(x) and lo = E4M3(x - hi).  A bf16 x has 8 significant
                        // bits and hi keeps the top 4, so x - hi is at most 8 times x's last bit,
                        // a multiple of it: x = hi + lo exactly wherever |x| >= 2^-2, which E4M3's
                        // smallest step (2^-9) reaches; below, the error is under 2^-10, 2^-17 of
                        // x_max.  Code row i takes hi and row N + i takes lo: the bytes of bf16
                        // half 0 and half 1 of row i, which the row's two threads (one per half,
                        // adjacent lanes) both read before either writes.
                        if (!tc::mbar_wait(q_full, qf_phase, abort_flag)) break;
                        qf_phase ^= 1;
                        const int hf = et & 1;
                        static_assert(N % (kEpiThreads / 2) == 0, "every lane takes the same rows");
                        for (int i = et >> 1; i < N; i += kEpiThreads / 2) {
                            const int sw = i & 7;   // 128-byte swizzle: chunk c of row i at c ^ (i & 7)
                            const uint8_t* src = qbuf + (size_t)hf * (N * 128) + (size_t)i * 128;
                            uint4 x[8];          // x[L]: dims 64 hf + 8 L .. + 7
                            float mx = 0.f;
#pragma unroll
                            for (int L = 0; L < 8; ++L) {
                                x[L] = *reinterpret_cast<const uint4*>(src + ((L ^ sw) * 16));
                                const uint32_t wv[4] = {x[L].x, x[L].y, x[L].z, x[L].w};
#pragma unroll
                                for (int qq = 0; qq < 4; ++qq) {
                                    const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[qq]));
                                    mx = fmaxf(mx, fmaxf(fabsf(f2.x), fabsf(f2.y)));
                                }
                            }
                            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                            const int e = mx > 0.f ? min(100, max(-100, floor_log2_f(mx) - 7)) : 0;
                            const float f = __uint_as_float((uint32_t)(127 - e) << 23);
                            uint32_t hi[16], lo[16];   // this thread's 64 codes of each, 4 per word
#pragma unroll
                            for (int L = 0; L < 8; ++L) {
                                const uint32_t wv[4] = {x[L].x, x[L].y, x[L].z, x[L].w};
#pragma unroll
                                for (int qq = 0; qq < 4; ++qq) {
                                    const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[qq]));
                                    const float2 xs = make_float2(f2.x * f, f2.y * f);
                                    const __nv_fp8x2_storage_t h = __nv_cvt_float2_to_fp8x2(xs, __NV_SATFINITE, __NV_E4M3);
                                    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(h, __NV_E4M3);
                                    const float2 hv = __half22float2(*reinterpret_cast<const __half2*>(&hr));
                                    const float2 rs = make_float2(xs.x - hv.x, xs.y - hv.y);
                                    const __nv_fp8x2_storage_t l = __nv_cvt_float2_to_fp8x2(rs, __NV_SATFINITE, __NV_E4M3);
                                    // codes 8 L + 2 qq and + 1 of this thread's 64
                                    if ((qq & 1) == 0) {
                                        hi[2 * L + (qq >> 1)] = (uint32_t)h;
                                        lo[2 * L + (qq >> 1)] = (uint32_t)l;
                                    } else {
                                        hi[2 * L + (qq >> 1)] |= (uint32_t)h << 16;
                                        lo[2 * L + (qq >> 1)] |= (uint32_t)l << 16;
                                    }
                                }
                            }
                            __syncwarp();   // both halves of row i are in registers
                            uint8_t* hrow = qbuf + (size_t)i * 128;
                            uint8_t* lrow = qbuf + (size_t)(N + i) * 128;   // (N + i) & 7 == i & 7
#pragma unroll
                            for (int j = 0; j < 4; ++j) {   // 16-code chunk 4 hf + j of the code rows
                                const int cc = ((4 * hf + j) ^ sw) * 16;
                                *reinterpret_cast<uint4*>(hrow + cc) =
                                    make_uint4(hi[4 * j], hi[4 * j + 1], hi[4 * j + 2], hi[4 * j + 3]);
                                *reinterpret_cast<uint4*>(lrow + cc) =
                                    make_uint4(lo[4 * j], lo[4 * j + 1], lo[4 * j + 2], lo[4 * j + 3]);
                            }
                            __syncwarp();
                            if (hf == 0) {
                                const int t = g * G + i / kHI;
                                w_s[i] = t < v.T_q ? w[(int64_t)t * kHI + (i % kHI)] *
                                                         __uint_as_float((uint32_t)(127 + e) << 23)
                                                   : 0.f;
                            }
                        }
                        tc::fence_async_smem();   // the query codes -> the tensor core
                    } else {
                        for (int i = et; i < N; i += kEpiThreads) {
                            const int t = g * G + i / kHI;
                            w_s[i] = t < v.T_q ? w[(int64_t)t * kHI + (i % kHI)] : 0.f;
                        }
                    }
                    if (kBs) {
                        // the group's query scale words into TMEM: column c, lane l holds query
                        // row (x head) 32c + l; each warp writes the copy in its own lane quarter
                        uint32_t qs[N / 32];
#pragma unroll
                        for (int c = 0; c < N / 32; ++c) {
                            const int i = 32 * c + lane;
                            qs[c] = g * G + i / kHI < v.T_q ? __ldg(q_scale + q_row0 + (int64_t)g * N + i) : 0u;
                        }
                        const uint32_t ta = tmem_base + ((uint32_t)(quarter * 32) << 16) + C::kSfbCol;
                        if constexpr (N == 64) tc::tmem_st2_u(ta, qs[0], qs[1]);
                        else tc::tmem_st4_u(ta, qs[0], qs[1], qs[2], qs[3]);
                        tc::tc_fence_before();
                    }
                    const GroupInfo gi = group_info(v, g, G, false);
                    seq_b = gi.b < 0 ? 0 : gi.b;
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        const int t = g * G + j;
                        row_pos[j] = -1;
                        if (t < v.T_q) {
                            RowInfo r = load_row(v, t);
                            if (r.pos >= 0 && r.b == gi.b) row_pos[j] = r.pos;
                        }
                    }
                    if (!epi_sync.sync(abort_flag)) break;   // the new weights are in place
                    if ((kF16 || kBs || kSp) && lane == 0) tc::mbar_arrive(q_ready);
                    cur = g;
                }
                if (!tc::mbar_wait(&acc_full[acc], acc_phase, abort_flag)) break;
                tc::tc_fence_after();
                const int s = kt * kBM + r_in_tile;
                const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * N;
                float kscale = 1.f;
                if (kSp) {
                    // the key's fp32 scale, bulk-copied with the codes into the stage's slot
                    // (waiting on the stage's own barrier makes the copy visible here)
                    if (!tc::mbar_wait(&full[es], ephase, abort_flag)) break;
                    kscale = reinterpret_cast<const float*>(kscl + (size_t)es * C::kScaleStageBytes)[r_in_tile];
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&sf_full[es]);
                    if (++es == (uint32_t)S) {
                        es = 0;
                        ephase ^= 1;
                    }
                } else if (kKeyScale) {
                    int pmax = -1;
#pragma unroll
                    for (int j = 0; j < G; ++j) pmax = max(pmax, row_pos[j]);
                    if (s <= pmax) {
                        const int64_t slot = epi_pshift >= 0 ? paged_slot_pow2(v, seq_b, s, epi_pshift)
                                                             : paged_slot(v, seq_b, s);
                        if (kMx) {
                            // the largest of the key's four block exponents; the converters
                            // scaled every block relative to it
                            const uint32_t wd = __ldg(static_cast<const uint32_t*>(k_scale) + slot);
                            const uint32_t emax = max(max(wd & 0xFFu, (wd >> 8) & 0xFFu),
                                                      max((wd >> 16) & 0xFFu, wd >> 24));
                            kscale = e8m0_to_f32(emax);
                        } else {
                            kscale = __ldg(static_cast<const float*>(k_scale) + slot);
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < G; ++j) {
                    if (j < jlo || j >= jhi) continue;
                    float a[64];
                    const float* wj = w_s + j * kHI;
                    float sc = 0.f;
                    if constexpr (G == 1) {
                        tc::tmem_ld32(taddr, a);
                        tc::tmem_ld32(taddr + 32, a + 32);
#pragma unroll
                        for (int h = 0; h < kHI; ++h) sc = fmaf(wj[h], fmaxf(a[h], 0.f), sc);
                    } else {
                        // several rows per tile: the epilogue bounds the kernel; one 64-column
                        // load and four partial sums (no 64-long dependent chain)
                        tc::tmem_ld64(taddr + j * kHI, a);
                        float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
                        for (int h = 0; h < kHI; h += 4) {
                            p0 = fmaf(wj[h], fmaxf(a[h], 0.f), p0);
                            p1 = fmaf(wj[h + 1], fmaxf(a[h + 1], 0.f), p1);
                            p2 = fmaf(wj[h + 2], fmaxf(a[h + 2], 0.f), p2);
                            p3 = fmaf(wj[h + 3], fmaxf(a[h + 3], 0.f), p3);
                        }
                        sc = (p0 + p1) + (p2 + p3);
                    }
                    if (kKeyScale) sc *= kscale;   // positive per-key scale factors out of the ReLU sum
                    if (s <= row_pos[j]) scores[(int64_t)(g * G + j) * ld + s] = sc;
                }
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&acc_empty[acc]);
                if (++acc == (uint32_t)C::kAcc) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
        } else if (kBs) {
            // ------------------------------------------------------------ key scales -> TMEM
            // warp 6 + i fills TMEM lane quarter (6 + i) % 4: column 4 x stage + c, lane l holds
            // the scale word of key 32c + l of the stage's tile (every quarter holds a copy)
            const int quarter = warp & 3;
            uint32_t stage = 0, phase = 0;
            for (int64_t f = f_begin; f < f_end; ++f) {
                if (!tc::mbar_wait(&full[stage], phase, abort_flag)) break;
                const uint32_t* wsc = reinterpret_cast<const uint32_t*>(kscl + (size_t)stage * C::kScaleStageBytes);
                tc::tmem_st4_u(tmem_base + ((uint32_t)(quarter * 32) << 16) + C::kSfaCol + 4 * stage,
                               wsc[lane], wsc[32 + lane], wsc[64 + lane], wsc[96 + lane]);
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&sf_full[stage]);
                if (++stage == (uint32_t)S) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        } else if (kFp8) {
            // ------------------------------------------------------------ FP8 -> bf16 converters
            // eight lanes widen one key row of the staging tile (16 codes each), four rows per warp
            // instruction, into the two 64-column swizzled halves of the bf16 tile the MMA reads
            // (e4m3 -> f16 -> bf16 is exact); a row's eight lanes read 128 contiguous bytes, so
            // the staging reads are free of bank conflicts
            constexpr int kRowsPerWarp = kBM / (C::kConv > 0 ? C::kConv : 4);   // 16 or 32
            const int cw = (tid - 192) >> 5;           // converter warp: rows kRowsPerWarp x cw ..
            const int c = lane & 7;                    // 16-code chunk of the row
            const int half = c >> 2;                   // which 64-column half it lands in
            const int chunk = (c & 3) * 2;             // first of its two 16-byte chunks there
            uint32_t stage = 0, phase = 0;
            uint32_t n = 0;
            for (int64_t f = f_begin; f < f_end; ++f, ++n) {
                if (!tc::mbar_wait(&raw_full[n % C::kR], (n / C::kR) & 1, abort_flag)) break;
                if (!tc::mbar_wait(&empty[stage], phase ^ 1, abort_flag)) break;
                const uint8_t* src = raw + (size_t)(n % C::kR) * (kBM * kDI);
                uint8_t* dst = tiles + (size_t)stage * kTileBytes + half * kHalfBytes;
#pragma unroll
                for (int i = 0; i < kRowsPerWarp / 4; ++i) {
                    const int r = kRowsPerWarp * cw + 4 * i + (lane >> 3);
                    const uint4 in = *reinterpret_cast<const uint4*>(src + r * 128 + c * 16);
                    const uint32_t words[4] = {in.x, in.y, in.z, in.w};
                    uint32_t outw[8];
                    if (kMx) {
                        // MXFP8: this lane's 16 codes lie in block c / 2 of the key.  Each code's
                        // sign, exponent and mantissa bits are placed in a bf16 (2^-120 times the
                        // code's value; a subnormal code becomes a bf16 subnormal), and one packed
                        // multiply by 2^(120 + E_block - E_max) gives code x 2^(E_block - E_max)
                        // exactly; 2^(E_max - 127) is left to the epilogue.  A block more than
                        // 2^246 below the key's largest is flushed to zero.
                        const uint32_t wd = reinterpret_cast<const uint32_t*>(
                            kscl + (size_t)(n % C::kR) * C::kScaleStageBytes)[r];
                        const int emax = (int)max(max(wd & 0xFFu, (wd >> 8) & 0xFFu),
                                                  max((wd >> 16) & 0xFFu, wd >> 24));
                        const int fe = 247 + (int)((wd >> (8 * (c >> 1))) & 0xFFu) - emax;
                        const uint32_t fb = fe > 0 ? (uint32_t)fe << 7 : 0u;
                        const uint32_t fb2 = fb | (fb << 16);
                        const __nv_bfloat162 f2 = *reinterpret_cast<const __nv_bfloat162*>(&fb2);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
#pragma unroll
                            for (int hlf = 0; hlf < 2; ++hlf) {
                                // codes 2*hlf and 2*hlf+1 of the word into the low and high bf16
                                const uint32_t t = __byte_perm(words[q], 0u, hlf ? 0x4342u : 0x4140u);
                                const uint32_t bits = ((t & 0x00800080u) << 8) | ((t & 0x007F007Fu) << 4);
                                const __nv_bfloat162 v2 =
                                    __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&bits), f2);
                                outw[q * 2 + hlf] = *reinterpret_cast<const uint32_t*>(&v2);
                            }
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
#pragma unroll
                            for (int hlf = 0; hlf < 2; ++hlf) {
                                // one conversion per code pair, straight to the f16 the MMA reads
                                const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)(words[q] >> (16 * hlf));
                                const __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
                                outw[q * 2 + hlf] = (uint32_t)h2.x | ((uint32_t)h2.y << 16);
                            }
                        }
                    }
                    uint8_t* rbase = dst + r * 128;
                    *reinterpret_cast<uint4*>(rbase + ((chunk ^ (r & 7)) * 16)) =
                        make_uint4(outw[0], outw[1], outw[2], outw[3]);
                    *reinterpret_cast<uint4*>(rbase + (((chunk + 1) ^ (r & 7)) * 16)) =
                        make_uint4(outw[4], outw[5], outw[6], outw[7]);
                }
                tc::fence_async_smem();
                tc::mbar_arrive(&raw_empty[n % C::kR]);
                tc::mbar_arrive(&full[stage]);
                if (++stage == (uint32_t)S) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, C::kTmemCols);
    }
    if (tid == 0 && *abort_flag) flag_status(v, HSA_DEV_TIMEOUT);
}

int num_sms() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <int G, bool kFp8, bool kMx, bool kBs = false, bool kSp = false>
cudaError_t launch_g(const IndexScoreArgs& a, cudaStream_t st) {
    using C = Cfg<G, kFp8, kMx, kBs, kSp>;
    const int box_rows = a.seq.page_size <= kBM ? a.seq.page_size : kBM;
    const uint64_t slots = (uint64_t)a.seq.num_pages * a.seq.page_size;
    CUtensorMap tk, tq;
    bool ok;
    if (kBs) {   // one 128-byte swizzled box per code row, for the keys and the queries
        ok = make_tensor_map_2d(&tk, a.k_cache, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, slots, kDI, kDI,
                                kDI, box_rows, CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_tensor_map_2d(&tq, a.q_I, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.seq.T_q * kHI,
                                kDI, kDI, kDI, C::N, CU_TENSOR_MAP_SWIZZLE_128B);
    } else {
        ok = kSp ? make_tensor_map_2d(&tk, a.k_cache, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, slots, kDI, kDI,
                                      kDI, box_rows, CU_TENSOR_MAP_SWIZZLE_128B)
           : kFp8 ? make_tensor_map_2d(&tk, a.k_cache, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, slots, kDI,
                                       kDI, kDI, box_rows, CU_TENSOR_MAP_SWIZZLE_NONE)
                  : make_tensor_map_2d(&tk, a.k_cache, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, slots,
                                       kDI, kDI * 2, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
        ok = ok && make_tensor_map_2d(&tq, a.q_I, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                      (uint64_t)a.seq.T_q * kHI, kDI, kDI * 2, 64, C::N,
                                      CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (!ok) return cudaErrorInvalidValue;
    auto kern = index_score_tc_kernel<G, kFp8, kMx, kBs, kSp>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
    if (e != cudaSuccess) return e;
    const int rows_per_launch = C::kMaxGroups * G;
    for (int t0 = 0; t0 < a.seq.T_q; t0 += rows_per_launch) {
        SeqView v = a.seq;
        v.T_q = min(rows_per_launch, a.seq.T_q - t0);
        v.q_seq += t0;
        v.q_pos += t0;
        const int64_t groups = ceil_div(v.T_q, G);
        const int grid = (int)std::min<int64_t>(num_sms(), std::max<int64_t>(1, groups * 64));
        e = launch_pdl(kern, dim3(grid), dim3(C::kThreads), C::kSmem, st, tk, tq, v, t0 * kHI,
                       a.w + (int64_t)t0 * kHI, a.k_scale, static_cast<const uint32_t*>(a.q_scale),
                       a.scores + (int64_t)t0 * a.ld, a.ld, box_rows);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

bool index_score_tc_supported(const IndexScoreArgs& a) {
    if (a.q_dtype == HSA_MXE4M3) {   // block-scaled MMA: MXFP8 queries need MXFP8 keys
        if (a.k_dtype != HSA_MXE4M3 || a.q_scale == nullptr || (reinterpret_cast<uintptr_t>(a.q_scale) & 15))
            return false;
    } else if (a.q_dtype != HSA_BF16 ||
               (a.k_dtype != HSA_BF16 && a.k_dtype != HSA_E4M3 && a.k_dtype != HSA_MXE4M3)) {
        return false;
    }
    if ((a.k_dtype == HSA_E4M3 || a.k_dtype == HSA_MXE4M3) && a.k_scale == nullptr) return false;
    if (a.k_dtype == HSA_MXE4M3 && (reinterpret_cast<uintptr_t>(a.k_scale) & 15)) return false;
    if (a.H_I != kHI || a.D_I != kDI) return false;
    const int p = a.seq.page_size;
    if (p % 8 != 0) return false;
    if (p <= kBM ? (kBM % p != 0) : (p % kBM != 0)) return false;
    if ((reinterpret_cast<uintptr_t>(a.q_I) & 15) || (reinterpret_cast<uintptr_t>(a.k_cache) & 15)) return false;
    if ((uint64_t)a.seq.num_pages * p >= (1ull << 31) || (uint64_t)a.seq.T_q * kHI >= (1ull << 31)) return false;
    return true;
}

cudaError_t launch_index_score_tc(const IndexScoreArgs& a, cudaStream_t st) {
    const bool fp8 = a.k_dtype == HSA_E4M3, mx = a.k_dtype == HSA_MXE4M3;
    if (a.q_dtype == HSA_MXE4M3)   // two query rows per tile at most (TMEM holds the scales too)
        return a.q_run % 2 == 0 ? launch_g<2, false, false, true>(a, st) : launch_g<1, false, false, true>(a, st);
    if (a.q_run % 4 == 0)
        return mx ? launch_g<4, true, true>(a, st) : fp8 ? launch_g<4, true, false>(a, st) : launch_g<4, false, false>(a, st);
    if (a.q_run % 2 == 0)
        return mx ? launch_g<2, true, true>(a, st) : fp8 ? launch_g<2, true, false>(a, st) : launch_g<2, false, false>(a, st);
    if (fp8 && (reinterpret_cast<uintptr_t>(a.k_scale) & 15) == 0) {   // split queries: scales by bulk copy
        if (a.q_run % 4 == 0) return launch_g<4, false, false, false, true>(a, st);
        if (a.q_run % 2 == 0) return launch_g<2, false, false, false, true>(a, st);
        return launch_g<1, false, false, false, true>(a, st);
    }
    return mx ? launch_g<1, true, true>(a, st) : fp8 ? launch_g<1, true, false>(a, st) : launch_g<1, false, false>(a, st);
}

}  // namespace hsa
