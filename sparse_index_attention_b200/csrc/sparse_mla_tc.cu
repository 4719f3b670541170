// sparse_mla_tc.cu -- tensor-core sparse MLA attention, 128 heads over a 512 + 64 latent cache.
//
// "Day 0 Inference Adaptation and Optimization for Hybrid Attention Models", "Sparse Attention
// Pipeline Optimization": read only the selected KV rows, block-wise fused attention; "Day-One
// Inference Adaptation for Very Large Hybrid-Attention Models", 3.2: partition by query,
// aggregate over the selected positions, stage them in shared memory.
//
// Per query row t the selected latent rows are gathered in tiles of 64 through the block table
// (cp.async by four producer warps: one warp instruction moves one row's 512-byte half, so every
// request is a full, coalesced line; the 128-byte / 64-byte swizzles the MMA expects are applied
// to the destination addresses) and every tile is shared by all 128 heads:
//     S = Q_t . KV^T            (M = 128 heads, N = 64 rows, K = 576)
//     P = online softmax(S)     (fp32, base-2 exponent, lazy rescale)
//     O += P . V                (M = 128 heads, N = 512 latent dims, K = 64 rows)
// The fp32 output accumulator O (128 x 512) alone fills the 512 TMEM columns of an SM, so a
// cluster of two CTAs splits the latent dims: CTA r owns value dims [256r, 256r + 256) and, for
// S, the matching 256 latent dims plus rope dims [512 + 32r, 544 + 32r).  Each CTA computes a
// partial S over its 288 dims, the pair swaps partial S through distributed shared memory
// (st.async that also completes the receiver's mbarrier transaction count), and both add the
// halves (fp32 addition commutes, so both hold the identical S and take identical softmax
// decisions).  Each CTA then accumulates its half of O.  No gathered byte and no MMA is
// duplicated between the two CTAs.
//
// Shared memory per CTA: the rope part of Q (8 KB, 64-byte swizzle), four KV stages of 64
// gathered rows (36 KB each: four 64-dim 128-byte-swizzled blocks + one 32-dim 64-byte-swizzled
// rope block; the stage is the K-major B operand of Q.KV^T and, read MN-major, the B operand of
// P.V), two 32 KB exchange buffers that receive the peer's partial S (fp32, laid out
// [4-column chunk][head][4] so that every warp-wide store and load covers 512 contiguous bytes),
// and the physical slots of the next 1024 selected entries.  Tensor memory: O (256 columns), two
// partial-S buffers (2 x 64 columns; P, bf16 pairs, overwrites the first half of its S buffer and
// is the TMEM A operand of P.V) and the latent part of Q (128 columns, the A operand of Q.KV^T).
//
// Pipeline per tile n: sender warps push partial S(n) to the peer as soon as Q.KV^T(n) is done,
// independent of the softmax, so the distributed-shared-memory hop overlaps the softmax of the
// previous tile, and the tensor core runs Q.KV^T(n+1) and P.V(n-1) while softmax(n) runs.  The
// peer may overwrite an exchange buffer only after this CTA's P.V of the tile that used it (MMA
// commit multicast to the peer), which is also what makes receiving tile n prove that P.V(n-2)
// has finished.  Measured on B200: one tcgen05.mma issues in about 60 cycles whatever its N, so
// Q.KV^T (18 MMAs of N = 64) costs more issue time than its flops; the cluster network moves the
// 32 KB exchange in about 1 us when warp stores are contiguous (1.8 us with one row per thread).
//
// (A TMA tile::gather4 version of the gather -- four 128-byte rows per instruction, 80 per tile
// and CTA -- delivered only about 0.75 TB/s here: the MMA warp waited on the gathered tiles for
// three quarters of the kernel.  Plain 16-byte asynchronous copies from 128 threads keep far more
// bytes in flight.)
//
// Warp roles: 0-3 producers (slot window + gather; warp w owns rows 16w..16w+15 of every tile),
// 4 MMA issuer, 5-12 softmax / epilogue (two threads per head h = TMEM lane h, 32 columns each;
// warps w and w + 4 share heads and swap tile maxima through a two-warp barrier), 13-16 senders
// (partial S to the peer).  Persistent: each cluster loops over query rows.
#include <algorithm>

#include "kernels.h"
#include "tc_common.cuh"

namespace hsa {

namespace {

constexpr int kH = 128;          // heads = MMA M = TMEM lanes
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kBN = 64;          // gathered rows per tile
constexpr int kStages = 4;
constexpr int kThreads = 544;   // 4 producer, 1 MMA, 8 softmax, 4 sender warps
constexpr int kSlotWin = 1024;   // selected entries whose slots are resolved at once (16 tiles)

constexpr int kQRopeBytes = kH * 64;               // 128 heads x 32 dims bf16, SW64
constexpr int kKvBlk = kBN * 128;                  // 64 rows x 64 dims
constexpr int kKvRope = kBN * 64;                  // 64 rows x 32 dims
constexpr int kStageBytes = 4 * kKvBlk + kKvRope;  // 36 KB
constexpr int kRecvBytes = kH * kBN * 4;           // 32 KB of fp32 partial S
constexpr int kOffStages = kQRopeBytes;
constexpr int kOffRecv = kOffStages + kStages * kStageBytes;
constexpr int kOffSlots = kOffRecv + 2 * kRecvBytes;
constexpr int kOffMasks = kOffSlots + 4 * kSlotWin;
constexpr int kOffXmax = kOffMasks + 8 * kStages;              // [2 tiles][2 halves][128] fp32
constexpr int kOffXsum = kOffXmax + 4 * 512;                   // [2 halves][128] fp32
constexpr int kOffBars = kOffXsum + 4 * 256;
constexpr int kKvRowBytes = kDqk * 2;   // 1152: bf16 latent ‖ rope
constexpr int kKv8RowBytes = kDv;       // 512: e4m3 latent codes (FP8 cache)
constexpr int kRopeRowBytes = 128;      // bf16 rope of the FP8 cache
constexpr size_t kSmem = 1024 + kOffBars + 256;
static_assert(kSmem <= 232448, "shared memory budget");
static_assert(kOffStages % 1024 == 0 && kStageBytes % 1024 == 0 && kOffRecv % 1024 == 0, "swizzle alignment");

constexpr uint32_t kTmemO = 0;       // 256 columns: this CTA's half of O
constexpr uint32_t kTmemS = 256;     // 2 x 64 columns: partial S, double-buffered
constexpr uint32_t kTmemQ = 384;     // 128 columns: this CTA's 256 latent dims of Q (bf16 pairs)
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdescQK = tc::idesc_bf16_f32(kH, kBN, 0, 0);
constexpr uint32_t kIdescPV = tc::idesc_bf16_f32(kH, 256, 0, 1);
constexpr float kRescaleLog2 = 8.f;  // rescale O only when the running max grows by > 2^8

struct Bars {
    uint64_t q_full;      // Q of the row in place: latent part in TMEM, rope part in smem (4 warps)
    uint64_t q_empty;     // last Q.KV^T of the row done
    uint64_t kv_full[kStages], kv_empty[kStages];
    uint64_t s_full[2], s_empty[2];
    uint64_t s_sent[2];     // the senders have read partial S of the buffer (P may overwrite it)
    uint64_t p_full;
    uint64_t pv_done;     // this CTA's P.V of a tile completed
    uint64_t peer_free[2];  // the peer's P.V of a tile of parity b completed (its buffer b is free)
    uint64_t recv_full[2];
    uint64_t o_ready, o_free;
    uint64_t pair_sync[4];  // the two softmax warps of a head quarter (maxima / row sums posted)
    uint32_t tmem;
    int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// 1 + the last index of idx row that is not -1 (0 if none), by a whole warp scanning from the end.
__device__ __forceinline__ int row_extent(const int32_t* __restrict__ idx_row, int K, int lane) {
    for (int k0 = ((K - 1) / 32) * 32; k0 >= 0; k0 -= 32) {
        const int k = k0 + lane;
        const bool used = k < K && __ldg(idx_row + k) != -1;
        const uint32_t m = __ballot_sync(0xffffffffu, used);
        if (m) return k0 + 32 - __clz(m);
    }
    return 0;
}

__device__ __forceinline__ int row_tiles(const SeqView& v, const int32_t* __restrict__ idx, int K, int t,
                                         int lane, RowInfo& r) {
    r = load_row(v, t);
    if (r.pos < 0) return 0;
    return (int)ceil_div(row_extent(idx + (int64_t)t * K, K, lane), kBN);
}

// kFp8Kv: the latent part of the cache is e4m3 codes with one fp32 scale per row and the rope part
// a separate bf16 array; the producers widen code x scale to bf16 on the way into the stage.
template <bool kFp8Kv>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
sparse_mla_tc_kernel(SeqView v,
                     const __nv_bfloat16* __restrict__ q, const uint8_t* __restrict__ kv_bytes,
                     const float* __restrict__ kv_scale, int kv_group, const uint8_t* __restrict__ rope_bytes,
                     int64_t rope_row_bytes, const int32_t* __restrict__ idx, int K,
                     float scale_log2, __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* q_rope = base;
    uint8_t* stages = base + kOffStages;
    uint8_t* recv = base + kOffRecv;
    int32_t* slots = reinterpret_cast<int32_t*>(base + kOffSlots);
    volatile uint64_t* masks = reinterpret_cast<volatile uint64_t*>(base + kOffMasks);
    float* xmax = reinterpret_cast<float*>(base + kOffXmax);
    float* xsum = reinterpret_cast<float*>(base + kOffXsum);
    Bars* bars = reinterpret_cast<Bars*>(base + kOffBars);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = tc::cluster_ctarank();
    const uint32_t peer = rank ^ 1u;
    const int cluster = blockIdx.x >> 1;
    const int n_clusters = gridDim.x >> 1;

    if (tid == 0) {
        tc::mbar_init(&bars->q_full, 8);
        tc::mbar_init(&bars->q_empty, 1);
        for (int i = 0; i < kStages; ++i) {
            // 128 producer threads when their copies land + 4 warps publishing their mask bits
            tc::mbar_init(&bars->kv_full[i], 128 + 4);
            tc::mbar_init(&bars->kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&bars->s_full[i], 1);
            tc::mbar_init(&bars->s_empty[i], 1);    // P.V of the tile whose P sits in the buffer
            tc::mbar_init(&bars->s_sent[i], 4);     // 4 sender warps
            tc::mbar_init(&bars->recv_full[i], 1);
        }
        tc::mbar_init(&bars->p_full, 8);
        tc::mbar_init(&bars->pv_done, 1);
        tc::mbar_init(&bars->peer_free[0], 1);
        tc::mbar_init(&bars->peer_free[1], 1);
        tc::mbar_init(&bars->o_ready, 1);
        tc::mbar_init(&bars->o_free, 8);
        for (int i = 0; i < 4; ++i) tc::mbar_init(&bars->pair_sync[i], 2);
        bars->abort = 0;
        tc::fence_barrier_init();
    }
    if (warp == 4) {
        tc::tmem_alloc(&bars->tmem, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync_all();  // the peer's barriers exist before anything remote touches them
    tc::tc_fence_after();
    const uint32_t tmem_base = bars->tmem;
    pdl_wait();              // the selection is the previous kernel's output
    pdl_trigger();

    if (warp < 4) {
        // ---------------------------------------------------------------- producers (gather)
        int32_t* my_slots = slots + warp * (kSlotWin / 4);   // this warp's 16 rows of 16 tiles
        uint16_t* masks16 = reinterpret_cast<uint16_t*>(const_cast<uint64_t*>(masks));
        uint32_t n = 0;
        bool stop = false;
        for (int t = cluster; t < v.T_q && !stop; t += n_clusters) {
            RowInfo r;
            const int ntiles = row_tiles(v, idx, K, t, lane, r);
            if (ntiles == 0) continue;
            const int32_t* idx_row = idx + (int64_t)t * K;
            for (int j = 0; j < ntiles; ++j, ++n) {
                if (j % (kSlotWin / kBN) == 0) {
                    // physical slots of this warp's rows for the next 32 tiles (-1: none), eight
                    // independent lookups per lane in flight at a time
#pragma unroll 1
                    for (int e0 = 0; e0 < kSlotWin / 4; e0 += 32 * 8) {
                        int32_t nn[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int e = e0 + lane + 32 * u;
                            const int k = (j + e / 16) * kBN + warp * 16 + (e % 16);
                            nn[u] = k < K ? __ldg(idx_row + k) : -1;
                        }
                        // the eight block-table reads are all in flight before any is used
                        bool bad_page = false, bad_pos = false;
                        int32_t sl[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const bool ok = nn[u] >= 0 && nn[u] <= r.pos;
                            bad_pos |= !ok && nn[u] != -1;
                            bool bp = false;
                            sl[u] = (int32_t)paged_slot_nb(v, r.b, ok ? nn[u] : 0, bp);
                            bad_page |= ok && bp;
                            if (!ok) sl[u] = -1;
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u) my_slots[e0 + lane + 32 * u] = sl[u];
                        if (bad_page) flag_status(v, HSA_DEV_BAD_PAGE);
                        if (bad_pos && rank == 0) flag_status(v, HSA_DEV_BAD_POS);
                    }
                    __syncwarp();
                }
                const uint32_t st = n % kStages;
                if (!tc::mbar_wait(&bars->kv_empty[st], ((n / kStages) & 1) ^ 1, abort_flag)) {
                    stop = true;
                    break;
                }
                const int32_t* ts = my_slots + (j % (kSlotWin / kBN)) * 16;
                uint8_t* sbase = stages + st * kStageBytes;
                if (!kFp8Kv) {
                    // latent half: one row per warp instruction, lane = 16-byte chunk
#pragma unroll 4
                    for (int k = 0; k < 16; ++k) {
                        const int row = warp * 16 + k;
                        const int32_t sl = ts[k];
                        const uint8_t* src = kv_bytes + (int64_t)(sl < 0 ? 0 : sl) * kKvRowBytes + 512 * rank + lane * 16;
                        uint8_t* dst = sbase + (lane >> 3) * kKvBlk + row * 128 + (((lane & 7) ^ (row & 7)) * 16);
                        tc::cp_async16(dst, src, sl < 0 ? 0u : 16u);
                    }
                } else {
                    // latent half: 256 codes per row, two rows per warp instruction (half-warp =
                    // row, lane = 16 codes); widened to bf16 (code x row scale, rounded once) and
                    // stored as the two 16-byte chunks the swizzled stage expects
                    const int sub = lane >> 4, cl = lane & 15;
                    // this lane's 16 codes lie in one scale group (groups are multiples of 16)
                    const int n_groups = kDv / kv_group, my_group = (256 * (int)rank + 16 * cl) / kv_group;
                    uint4 raw[8];
                    float scl[8];
#pragma unroll
                    for (int k2 = 0; k2 < 8; ++k2) {
                        const int32_t sl = ts[2 * k2 + sub];
                        raw[k2] = sl < 0 ? make_uint4(0u, 0u, 0u, 0u)
                                         : __ldg(reinterpret_cast<const uint4*>(kv_bytes + (int64_t)sl * kKv8RowBytes + 256 * rank) + cl);
                        scl[k2] = sl < 0 ? 0.f : __ldg(kv_scale + (int64_t)sl * n_groups + my_group);
                    }
#pragma unroll
                    for (int k2 = 0; k2 < 8; ++k2) {
                        const int row = warp * 16 + 2 * k2 + sub;
                        const uint32_t words[4] = {raw[k2].x, raw[k2].y, raw[k2].z, raw[k2].w};
                        uint32_t outw[8];
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq) {
#pragma unroll
                            for (int hlf = 0; hlf < 2; ++hlf) {
                                const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)(words[qq] >> (16 * hlf));
                                const float2 f2 = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3)));
                                const __nv_bfloat162 b2 = __floats2bfloat162_rn(f2.x * scl[k2], f2.y * scl[k2]);
                                outw[qq * 2 + hlf] = *reinterpret_cast<const uint32_t*>(&b2);
                            }
                        }
                        // codes 16cl..16cl+15 are dims of 16-byte chunks 2cl and 2cl+1
                        uint8_t* rbase = sbase + (cl >> 2) * kKvBlk + row * 128;
                        *reinterpret_cast<uint4*>(rbase + ((((2 * cl) & 7) ^ (row & 7)) * 16)) =
                            make_uint4(outw[0], outw[1], outw[2], outw[3]);
                        *reinterpret_cast<uint4*>(rbase + ((((2 * cl + 1) & 7) ^ (row & 7)) * 16)) =
                            make_uint4(outw[4], outw[5], outw[6], outw[7]);
                    }
                    tc::fence_async_smem();   // these generic stores -> the tensor core
                }
                // rope half: 4 chunks per row, 8 rows per instruction
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int row = warp * 16 + 8 * h2 + (lane >> 2);
                    const int cc = lane & 3;
                    const int32_t sl = ts[8 * h2 + (lane >> 2)];
                    const uint8_t* src = rope_bytes + (int64_t)(sl < 0 ? 0 : sl) * rope_row_bytes + 64 * rank + cc * 16;
                    uint8_t* dst = sbase + 4 * kKvBlk + row * 64 + ((cc ^ ((row >> 1) & 3)) * 16);
                    tc::cp_async16(dst, src, sl < 0 ? 0u : 16u);
                }
                // the stage is complete when every thread's copies have landed (hardware arrive)
                // and every warp has published its rows' validity bits
                tc::cp_async_arrive_noinc(&bars->kv_full[st]);
                const uint32_t vm = __ballot_sync(0xffffffffu, lane < 16 && ts[lane & 15] >= 0) & 0xFFFFu;
                __syncwarp();             // orders the warp's generic stores before lane 0's arrive
                if (lane == 0) {
                    masks16[st * 4 + warp] = (uint16_t)vm;
                    tc::mbar_arrive(&bars->kv_full[st]);
                }
            }
        }
        tc::cp_async_wait<0>();   // nothing of this thread still in flight when the CTA leaves
    } else if (warp == 4) {
        // ---------------------------------------------------------------- MMA issuer
        const uint32_t qr_addr = tc::smem_u32(q_rope);
        uint32_t n = 0, qr = 0, rows_done = 0;
        bool stop = false;
        auto pv = [&](uint32_t m, bool first) -> bool {
            if (!tc::mbar_wait(&bars->p_full, m & 1, abort_flag)) return false;
            if (first && !tc::mbar_wait(&bars->o_free, (rows_done & 1) ^ 1, abort_flag)) return false;
            tc::tc_fence_after();
            if (lane == 0) {
                const uint32_t p_tmem = tmem_base + kTmemS + (m & 1) * kBN;   // P (bf16 pairs) over S
                const uint32_t v_addr = tc::smem_u32(stages + (m % kStages) * kStageBytes);
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    tc::mma_bf16_tmem_a(tmem_base + kTmemO, p_tmem + 8 * kk,
                                        tc::sw128_desc(v_addr + kk * 2048, kKvBlk, 1024), kIdescPV,
                                        (first && kk == 0) ? 0u : 1u);
                tc::mma_commit(&bars->kv_empty[m % kStages]);
                tc::mma_commit(&bars->s_empty[m & 1]);
                tc::mma_commit(&bars->pv_done);
                tc::mma_commit_multicast(&bars->peer_free[m & 1], (uint16_t)(1u << peer));
            }
            __syncwarp();
            return true;
        };
        for (int t = cluster; t < v.T_q && !stop; t += n_clusters) {
            RowInfo r;
            const int ntiles = row_tiles(v, idx, K, t, lane, r);
            if (ntiles == 0) continue;
            if (!tc::mbar_wait(&bars->q_full, qr & 1, abort_flag)) break;
            ++qr;
            for (int j = 0; j < ntiles; ++j, ++n) {
                const uint32_t st = n % kStages, sb = n & 1;
                if (!tc::mbar_wait(&bars->kv_full[st], (n / kStages) & 1, abort_flag) ||
                    !tc::mbar_wait(&bars->s_empty[sb], ((n >> 1) & 1) ^ 1, abort_flag)) {
                    stop = true;
                    break;
                }
                tc::fence_async_smem();   // the gathered tile (generic-proxy copies) -> tensor core
                tc::tc_fence_after();
                if (lane == 0) {
                    const uint32_t kv_addr = tc::smem_u32(stages + st * kStageBytes);
                    const uint32_t d = tmem_base + kTmemS + sb * kBN;
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        tc::mma_bf16_tmem_a(d, tmem_base + kTmemQ + 8 * k,
                                            tc::sw128_desc(kv_addr + (k >> 2) * kKvBlk + (k & 3) * 32, 16, 1024),
                                            kIdescQK, k ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        tc::mma_bf16(d, tc::sw64_desc(qr_addr + kk * 32, 512),
                                     tc::sw64_desc(kv_addr + 4 * kKvBlk + kk * 32, 512), kIdescQK, 1u);
                    tc::mma_commit(&bars->s_full[sb]);
                    if (j == ntiles - 1) tc::mma_commit(&bars->q_empty);
                }
                __syncwarp();
                if (j > 0 && !pv(n - 1, j == 1)) {
                    stop = true;
                    break;
                }
            }
            if (stop || !pv(n - 1, ntiles == 1)) break;
            if (lane == 0) tc::mma_commit(&bars->o_ready);
            __syncwarp();
            ++rows_done;
        }
    } else if (warp < 13) {
        // ---------------------------------------------------------------- softmax
        // Two threads per head: warps 5-8 take columns 0..31 of every tile and output dims
        // 0..127 of this CTA's half, warps 9-12 columns 32..63 and dims 128..255.  They combine
        // their tile maxima through xmax (double-buffered by tile parity) and their row sums
        // through xsum at the end of a row.
        const int h = (warp & 3) * 32 + lane;          // head = TMEM lane
        const int half = (warp - 5) >> 2;              // which 32 columns / 128 output dims
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t col = (uint32_t)(32 * half);
        uint32_t n = 0, rows_done = 0;
        bool stop = false;
        tc::WarpSetSync pair_sync{&bars->pair_sync[(warp - 5) & 3], 0};   // warps w and w + 4

        // next row (t0, t0 + n_clusters, ...) with work; rows without any selection are written
        // here directly (output 0, lse -inf)
        auto next_row = [&](int t0, int& ntiles, RowInfo& r) -> int {
            for (int t = t0; t < v.T_q; t += n_clusters) {
                ntiles = row_tiles(v, idx, K, t, lane, r);
                if (ntiles > 0) return t;
                __nv_bfloat16* orow = out + ((int64_t)t * kH + h) * kDv + 256 * rank + 128 * half;
                for (int c = 0; c < 128; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
                if (lse != nullptr && rank == 0 && half == 0) lse[(int64_t)t * kH + h] = -INFINITY;
            }
            return -1;
        };
        // Q row t: this CTA's 256 latent dims into TMEM (lane h, columns 384.. as bf16 pairs) and
        // its 32 rope dims into shared memory (64-byte swizzle: chunk c of row h at c ^ ((h>>1)&3));
        // each of the two threads of a head moves half of it
        auto load_q = [&](int t) {
            const uint4* srcr = reinterpret_cast<const uint4*>(q + ((int64_t)t * kH + h) * kDqk + 512 + 32 * rank);
#pragma unroll
            for (int c = 2 * half; c < 2 * half + 2; ++c)
                *reinterpret_cast<uint4*>(q_rope + h * 64 + ((c ^ ((h >> 1) & 3)) * 16)) = __ldg(srcr + c);
            tc::fence_async_smem();
            const uint4* src = reinterpret_cast<const uint4*>(q + ((int64_t)t * kH + h) * kDqk + 256 * rank);
#pragma unroll 1
            for (int c = 2 * half; c < 2 * half + 2; ++c) {
                uint32_t w[32];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 x = __ldg(src + 8 * c + i);
                    w[4 * i] = x.x;
                    w[4 * i + 1] = x.y;
                    w[4 * i + 2] = x.z;
                    w[4 * i + 3] = x.w;
                }
                tc::tmem_st32_u(tmem_base + lane_off + kTmemQ + 32 * c, w);
            }
            tc::tmem_st_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->q_full);
        };
        int ntiles = 0;
        RowInfo r;
        int t = next_row(cluster, ntiles, r);
        if (t >= 0) load_q(t);
        while (t >= 0 && !stop) {
            float m_used = -INFINITY, l = 0.f;
            int t_next = -1, ntiles_next = 0;
            RowInfo r_next;
            for (int j = 0; j < ntiles; ++j, ++n) {
                const uint32_t b = n & 1, st = n % kStages;
                // ---- softmax(n), columns [col, col + 32)
                // own partial S(n) is complete once the senders have read it (s_sent), which
                // also frees its columns for P; it is loaded while the peer's half is in flight
                if (!tc::mbar_wait(&bars->kv_full[st], (n / kStages) & 1, abort_flag) ||
                    !tc::mbar_wait(&bars->s_sent[b], (n >> 1) & 1, abort_flag)) {
                    stop = true;
                    break;
                }
                const uint32_t valid = (uint32_t)(masks[st] >> col);
                tc::tc_fence_after();
                float s[32];
                tc::tmem_ld32(tmem_base + lane_off + kTmemS + b * kBN + col, s);
                tc::tmem_ld_wait();
                if (!tc::mbar_wait_cluster(&bars->recv_full[b], (n >> 1) & 1, abort_flag)) {
                    stop = true;
                    break;
                }
                const float4* other = reinterpret_cast<const float4*>(recv + b * kRecvBytes) + h;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 o = other[(8 * half + i) * kH];
                    s[4 * i] += o.x;
                    s[4 * i + 1] += o.y;
                    s[4 * i + 2] += o.z;
                    s[4 * i + 3] += o.w;
                }
                if (__any_sync(0xffffffffu, valid != 0xffffffffu)) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (!((valid >> i) & 1u)) s[i] = -INFINITY;
                }
                float mt = s[0];
#pragma unroll
                for (int i = 1; i < 32; ++i) mt = fmaxf(mt, s[i]);
                mt = mt == -INFINITY ? -INFINITY : mt * scale_log2;   // tile max in base-2 units
                xmax[(n & 1) * 256 + half * 128 + h] = mt;
                if (!pair_sync.sync(abort_flag)) {  // both halves' maxima posted
                    stop = true;
                    break;
                }
                mt = fmaxf(mt, xmax[(n & 1) * 256 + (half ^ 1) * 128 + h]);
                // lazy rescale: a head whose running max grew by more than 2^8 rescales O and l
                // to the new max (both threads of the head take the same decision; the TMEM
                // accesses are warp-wide)
                float m_new = m_used;
                if (mt != -INFINITY) {
                    if (m_used == -INFINITY) m_used = m_new = mt;
                    else if (mt > m_used + kRescaleLog2) m_new = mt;
                }
                if (__any_sync(0xffffffffu, m_new != m_used)) {
                    // O holds P.V up to tile n-1 once that P.V completed
                    if (!tc::mbar_wait(&bars->pv_done, (n - 1) & 1, abort_flag)) {
                        stop = true;
                        break;
                    }
                    tc::tc_fence_after();
                    const float alpha = m_new != m_used ? tc::fast_exp2(m_used - m_new) : 1.f;
                    m_used = m_new;
                    l *= alpha;
#pragma unroll 1
                    for (int c = 128 * half; c < 128 * half + 128; c += 32) {
                        float o[32];
                        tc::tmem_ld32(tmem_base + lane_off + kTmemO + c, o);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] *= alpha;
                        tc::tmem_st32(tmem_base + lane_off + kTmemO + c, o);
                    }
                    tc::tmem_st_wait();
                }
                // p = 2^(s * scale_log2 - m): one FFMA per element (masked entries are -inf -> 0);
                // a head with nothing valid so far (m = -inf) contributes zeros
                const float mneg = m_used == -INFINITY ? 0.f : -m_used;
                const bool none = m_used == -INFINITY;
                float ps[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float p0 = none ? 0.f : tc::fast_exp2(fmaf(s[i], scale_log2, mneg));
                    const float p1 = none ? 0.f : tc::fast_exp2(fmaf(s[i + 1], scale_log2, mneg));
                    ps[(i >> 1) & 3] += p0 + p1;
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                    pk[i / 2] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
                // P over this thread's 32 columns of the S buffer: rows 32*half.. -> 16 columns of
                // bf16 pairs (the senders have read partial S, and the other half of the head read
                // its columns before the maxima were exchanged)
                tc::tmem_st16_u(tmem_base + lane_off + kTmemS + b * kBN + 16 * half, pk);
                tc::tmem_st_wait();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->p_full);
                // ---- last tile of the row: put the next row's Q in place
                if (j + 1 == ntiles) {
                    t_next = next_row(t + n_clusters, ntiles_next, r_next);
                    if (t_next >= 0) {
                        if (!tc::mbar_wait(&bars->q_empty, rows_done & 1, abort_flag)) {
                            stop = true;
                            break;
                        }
                        tc::tc_fence_after();
                        load_q(t_next);
                    }
                }
            }
            if (stop) break;
            // ---- row epilogue: O / l -> bf16 -> global (this thread: 128 of the 256 dims)
            xsum[half * 128 + h] = l;
            if (!tc::mbar_wait(&bars->o_ready, rows_done & 1, abort_flag) || !pair_sync.sync(abort_flag)) break;
            tc::tc_fence_after();
            const float l_all = l + xsum[(half ^ 1) * 128 + h];
            __nv_bfloat16* orow = out + ((int64_t)t * kH + h) * kDv + 256 * rank + 128 * half;
            const float inv_l = l_all > 0.f ? 1.f / l_all : 0.f;
#pragma unroll 1
            for (int c = 0; c < 128; c += 32) {
                float o[32];
                tc::tmem_ld32(tmem_base + lane_off + kTmemO + 128 * half + c, o);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                    uint32_t w4[4];
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(o[i + 2 * qq] * inv_l, o[i + 2 * qq + 1] * inv_l);
                        w4[qq] = *reinterpret_cast<const uint32_t*>(&b2);
                    }
                    *reinterpret_cast<uint4*>(orow + c + i) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->o_free);
            if (lse != nullptr && rank == 0 && half == 0)
                lse[(int64_t)t * kH + h] = l_all > 0.f ? (m_used + log2f(l_all)) * 0.69314718055994531f : -INFINITY;
            ++rows_done;
            t = t_next;
            ntiles = ntiles_next;
            r = r_next;
        }
    } else {
        // ---------------------------------------------------------------- senders
        // Warps 13-16 (one per TMEM lane quarter, thread = head) push every partial S tile to
        // the peer's exchange buffer as soon as its Q.KV^T completes, so the distributed-memory
        // hop never waits behind a softmax.
        const int h = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        uint32_t peer_recv[2], peer_bar[2];
        for (int b = 0; b < 2; ++b) {
            peer_recv[b] = tc::mapa_shared(tc::smem_u32(recv + b * kRecvBytes), peer);
            peer_bar[b] = tc::mapa_shared(tc::smem_u32(&bars->recv_full[b]), peer);
        }
        uint32_t m = 0;
        bool stop = false;
        for (int t = cluster; t < v.T_q && !stop; t += n_clusters) {
            RowInfo r;
            const int ntiles = row_tiles(v, idx, K, t, lane, r);
            for (int j = 0; j < ntiles; ++j, ++m) {
                const uint32_t b = m & 1;
                if (!tc::mbar_wait(&bars->s_full[b], (m >> 1) & 1, abort_flag)) {
                    stop = true;
                    break;
                }
                tc::tc_fence_after();
                float sv[kBN];
                tc::tmem_ld32(tmem_base + lane_off + kTmemS + b * kBN, sv);
                tc::tmem_ld32(tmem_base + lane_off + kTmemS + b * kBN + 32, sv + 32);
                tc::tmem_ld_wait();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->s_sent[b]);
                // the peer's P.V(m-2) has released its buffer b.  One barrier per buffer: the
                // peer cannot complete P.V(m) before it receives this tile, so the barrier is
                // never two phases ahead of this wait (with a single barrier for both buffers it
                // could be, since the peer may finish P.V(m-1) first, and a parity wait would
                // then alias).
                if (m >= 2 && !tc::mbar_wait(&bars->peer_free[b], ((m - 2) >> 1) & 1, abort_flag)) {
                    stop = true;
                    break;
                }
                if (warp == 13 && lane == 0) tc::mbar_arrive_expect_tx(&bars->recv_full[b], kRecvBytes);
                // chunk i (columns 4i..4i+3) of every head lies at [i][head]: each warp instruction
                // writes 512 contiguous bytes, which the cluster network moves about twice as fast
                // as one row per thread
                const uint32_t dst = peer_recv[b] + h * 16;
#pragma unroll
                for (int i = 0; i < kBN / 4; ++i)
                    tc::st_async_v4(dst + i * (kH * 16), peer_bar[b], __float_as_uint(sv[4 * i]),
                                    __float_as_uint(sv[4 * i + 1]), __float_as_uint(sv[4 * i + 2]),
                                    __float_as_uint(sv[4 * i + 3]));
            }
        }
        // the peer's last two P.V commits arrive here; take them before leaving
        if (!stop) {
            if (m >= 2) tc::mbar_wait(&bars->peer_free[(m - 2) & 1], ((m - 2) >> 1) & 1, abort_flag);
            if (m >= 1) tc::mbar_wait(&bars->peer_free[(m - 1) & 1], ((m - 1) >> 1) & 1, abort_flag);
        }
    }
    __syncwarp();
    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync_all();
    if (warp == 4) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, kTmemCols);
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

}  // namespace

bool sparse_mla_tc_supported(const SparseMlaArgs& a) {
    if (a.q_dtype != HSA_BF16 || a.out_dtype != HSA_BF16) return false;
    if (a.kv_dtype != HSA_BF16 && a.kv_dtype != HSA_E4M3) return false;
    if (a.kv_dtype == HSA_E4M3 && (a.kv_scale == nullptr || a.kv_rope == nullptr)) return false;
    if (a.kv_dtype == HSA_E4M3 && (a.kv_scale_group < 16 || a.kv_scale_group % 16 || kDv % a.kv_scale_group))
        return false;
    if (a.H != kH || a.D_qk != kDqk || a.D_v != kDv) return false;
    if (!(a.softmax_scale > 0.f)) return false;   // the kernel takes tile maxima on unscaled S
    auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    if (!al(a.q) || !al(a.kv) || !al(a.out)) return false;
    if (a.kv_dtype == HSA_E4M3 && (!al(a.kv_rope) || (reinterpret_cast<uintptr_t>(a.kv_scale) & 3))) return false;
    if ((uint64_t)a.seq.T_q * kH >= (1ull << 31)) return false;
    if ((uint64_t)a.seq.num_pages * a.seq.page_size >= (1ull << 31)) return false;
    return true;
}

size_t sparse_mla_tc_workspace(int32_t, int32_t) { return 0; }

cudaError_t launch_sparse_mla_tc(const SparseMlaArgs& a, cudaStream_t st) {
    if (a.seq.T_q == 0) return cudaSuccess;
    const bool fp8 = a.kv_dtype == HSA_E4M3;
    auto kern = fp8 ? sparse_mla_tc_kernel<true> : sparse_mla_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    const int clusters = std::max(1, std::min(a.seq.T_q, num_sms() / 2));
    const float scale_log2 = a.softmax_scale * 1.4426950408889634f;
    const uint8_t* kv = reinterpret_cast<const uint8_t*>(a.kv);
    // the bf16 cache packs the rope dims after the latent ones in each 1152-byte row
    const uint8_t* rope = fp8 ? reinterpret_cast<const uint8_t*>(a.kv_rope) : kv + 2 * kDv;
    const int64_t rope_row = fp8 ? kRopeRowBytes : kKvRowBytes;
    e = launch_pdl(kern, dim3(2 * clusters), dim3(kThreads), kSmem, st, a.seq,
                   reinterpret_cast<const __nv_bfloat16*>(a.q), kv, fp8 ? a.kv_scale : nullptr,
                   fp8 ? a.kv_scale_group : kDv, rope, rope_row,
                   a.idx, a.K, scale_log2, reinterpret_cast<__nv_bfloat16*>(a.out), a.lse);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace hsa
