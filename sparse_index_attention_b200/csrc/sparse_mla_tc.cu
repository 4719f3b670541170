// sparse_mla_tc.cu -- tensor-core sparse MLA attention, 128 heads over a 512 + 64 latent cache.
//
// "Day 0 Inference Adaptation and Optimization for Hybrid Attention Models", "Sparse Attention
// Pipeline Optimization": read only the selected KV rows, block-wise fused attention; "Day-One
// Inference Adaptation for Very Large Hybrid-Attention Models", 3.2: partition by query,
// aggregate over the selected positions, stage them in shared memory.
//
// Per query row t the selected latent rows are gathered in tiles of 64 (TMA tile::gather4
// through the block table) and every tile is shared by all 128 heads:
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
// Shared memory per CTA: Q (72 KB: four 64-dim 128-byte-swizzled blocks + one 32-dim
// 64-byte-swizzled rope block), three KV stages of 64 rows (36 KB each, same block structure;
// the stage is the K-major B operand of Q.KV^T and, read MN-major, the B operand of P.V), and a
// 32 KB exchange buffer that receives the peer's partial S; after it is read, P (bf16, 16 KB)
// is written over it.  Ordering needs no extra barrier: the peer only sends tile n after this
// CTA's P.V of tile n-1 completed (its MMA commit is multicast to the peer), so receiving tile n
// also proves that the previous P is no longer in use.
//
// Warp roles: 0 TMA producer (gather), 1 MMA issuer, 2-5 softmax / exchange / epilogue (thread h
// owns head h = TMEM lane h).  Persistent: each cluster loops over query rows.
#include <algorithm>

#include "kernels.h"
#include "tc_common.cuh"

namespace hsa {

namespace {

constexpr int kH = 128;          // heads = MMA M = TMEM lanes
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kBN = 64;          // gathered rows per tile
constexpr int kStages = 3;
constexpr int kThreads = 192;

constexpr int kQBlk = kH * 128;                    // 128 heads x 64 dims bf16, SW128
constexpr int kQRope = kH * 64;                    // 128 heads x 32 dims bf16, SW64
constexpr int kQBytes = 4 * kQBlk + kQRope;        // 72 KB
constexpr int kKvBlk = kBN * 128;                  // 64 rows x 64 dims
constexpr int kKvRope = kBN * 64;                  // 64 rows x 32 dims
constexpr int kStageBytes = 4 * kKvBlk + kKvRope;  // 36 KB
constexpr int kOffStages = kQBytes;
constexpr int kOffRecv = kOffStages + kStages * kStageBytes;
constexpr int kRecvBytes = kH * kBN * 4;           // 32 KB of fp32 partial S
constexpr int kOffBars = kOffRecv + kRecvBytes;
constexpr size_t kSmem = 1024 + kOffBars + 256;
static_assert(kSmem <= 232448, "shared memory budget");

constexpr uint32_t kTmemO = 0;       // 256 columns: this CTA's half of O
constexpr uint32_t kTmemS = 256;     // 2 x 64 columns: partial S, double-buffered
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdescQK = tc::idesc_bf16_f32(kH, kBN, 0, 0);
constexpr uint32_t kIdescPV = tc::idesc_bf16_f32(kH, 256, 0, 1);
constexpr float kRescaleLog2 = 8.f;  // rescale O only when the running max grows by > 2^8

struct Bars {
    uint64_t q_full, q_empty;
    uint64_t kv_full[kStages], kv_empty[kStages];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full;
    uint64_t peer_free;   // the peer's P.V of the previous tile is done (its buffer is free)
    uint64_t recv_full;   // the peer's partial S of this tile has landed here
    uint64_t o_ready, o_free;
    uint32_t tmem;
    int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// Number of leading entries of idx row t that can hold a selection (1 + last index != -1),
// computed by a whole warp scanning from the end.
__device__ __forceinline__ int row_extent(const int32_t* __restrict__ idx_row, int K, int lane) {
    for (int k0 = ((K - 1) / 32) * 32; k0 >= 0; k0 -= 32) {
        const int k = k0 + lane;
        const bool used = k < K && __ldg(idx_row + k) != -1;
        const uint32_t m = __ballot_sync(0xffffffffu, used);
        if (m) return k0 + 32 - __clz(m);
    }
    return 0;
}

// Physical slot of selected entry k of a row (0 for padding or an invalid entry, which the
// softmax masks out).
__device__ __forceinline__ int32_t entry_slot(const SeqView& v, const int32_t* __restrict__ idx_row,
                                              int K, int k, int b, int pos) {
    if (k >= K) return 0;
    const int n = __ldg(idx_row + k);
    if (n < 0 || n > pos) return 0;
    return (int32_t)paged_slot(v, b, n);
}

__device__ __forceinline__ bool entry_valid(const int32_t* __restrict__ idx_row, int K, int k, int pos,
                                            const SeqView& v, bool flag) {
    if (k >= K) return false;
    const int n = __ldg(idx_row + k);
    if (n == -1) return false;
    if (n < 0 || n > pos) {
        if (flag) flag_status(v, HSA_DEV_BAD_POS);
        return false;
    }
    return true;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
sparse_mla_tc_kernel(const __grid_constant__ CUtensorMap tm_q_lat, const __grid_constant__ CUtensorMap tm_q_rope,
                     const __grid_constant__ CUtensorMap tm_kv_lat, const __grid_constant__ CUtensorMap tm_kv_rope,
                     SeqView v, const int32_t* __restrict__ idx, int K, float scale_log2,
                     __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* qs = base;
    uint8_t* stages = base + kOffStages;
    uint8_t* recv = base + kOffRecv;
    Bars* bars = reinterpret_cast<Bars*>(base + kOffBars);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = tc::cluster_ctarank();
    const uint32_t peer = rank ^ 1u;
    const int cluster = blockIdx.x >> 1;
    const int n_clusters = gridDim.x >> 1;

    if (tid == 0) {
        tc::mbar_init(&bars->q_full, 1);
        tc::mbar_init(&bars->q_empty, 1);
        for (int i = 0; i < kStages; ++i) {
            tc::mbar_init(&bars->kv_full[i], 1);
            tc::mbar_init(&bars->kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&bars->s_full[i], 1);
            tc::mbar_init(&bars->s_empty[i], 4);
        }
        tc::mbar_init(&bars->p_full, 4);
        tc::mbar_init(&bars->peer_free, 1);
        tc::mbar_init(&bars->recv_full, 1);
        tc::mbar_init(&bars->o_ready, 1);
        tc::mbar_init(&bars->o_free, 4);
        bars->abort = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(&bars->tmem, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync_all();  // the peer's barriers exist before anything remote touches them
    tc::tc_fence_after();
    const uint32_t tmem_base = bars->tmem;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer (TMA)
        if (lane == 0) {
            tc::tma_prefetch_desc(&tm_q_lat);
            tc::tma_prefetch_desc(&tm_q_rope);
            tc::tma_prefetch_desc(&tm_kv_lat);
            tc::tma_prefetch_desc(&tm_kv_rope);
        }
        uint32_t n = 0, qr = 0;
        bool stop = false;
        for (int t = cluster; t < v.T_q && !stop; t += n_clusters) {
            const RowInfo r = load_row(v, t);
            const int32_t* idx_row = idx + (int64_t)t * K;
            const int ntiles = r.pos < 0 ? 0 : (int)ceil_div(row_extent(idx_row, K, lane), kBN);
            if (ntiles == 0) continue;
            if (qr > 0 && !tc::mbar_wait(&bars->q_empty, (qr - 1) & 1, abort_flag)) break;
            if (lane == 0) {
                tc::mbar_arrive_expect_tx(&bars->q_full, kQBytes);
                for (int kb = 0; kb < 4; ++kb)
                    tc::tma_load_2d(qs + kb * kQBlk, &tm_q_lat, &bars->q_full, 256 * rank + 64 * kb, t * kH);
                tc::tma_load_2d(qs + 4 * kQBlk, &tm_q_rope, &bars->q_full, 512 + 32 * rank, t * kH);
            }
            ++qr;
            for (int j = 0; j < ntiles; ++j, ++n) {
                const uint32_t st = n % kStages;
                if (!tc::mbar_wait(&bars->kv_empty[st], ((n / kStages) & 1) ^ 1, abort_flag)) {
                    stop = true;
                    break;
                }
                const int k0 = j * kBN;
                const int32_t slot_a = entry_slot(v, idx_row, K, k0 + lane, r.b, r.pos);
                const int32_t slot_b = entry_slot(v, idx_row, K, k0 + 32 + lane, r.b, r.pos);
                uint8_t* sbase = stages + st * kStageBytes;
                if (lane == 0) tc::mbar_arrive_expect_tx(&bars->kv_full[st], kStageBytes);
#pragma unroll 1
                for (int g = 0; g < kBN / 4; ++g) {
                    const int32_t src = g < 8 ? slot_a : slot_b;
                    const int l0 = (4 * g) & 31;
                    const int32_t y0 = __shfl_sync(0xffffffffu, src, l0);
                    const int32_t y1 = __shfl_sync(0xffffffffu, src, l0 + 1);
                    const int32_t y2 = __shfl_sync(0xffffffffu, src, l0 + 2);
                    const int32_t y3 = __shfl_sync(0xffffffffu, src, l0 + 3);
                    if (lane == 0) {
                        for (int kb = 0; kb < 4; ++kb)
                            tc::tma_gather4(sbase + kb * kKvBlk + g * 512, &tm_kv_lat, &bars->kv_full[st],
                                            256 * rank + 64 * kb, y0, y1, y2, y3);
                        tc::tma_gather4(sbase + 4 * kKvBlk + g * 256, &tm_kv_rope, &bars->kv_full[st],
                                        512 + 32 * rank, y0, y1, y2, y3);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        const uint32_t q_addr = tc::smem_u32(qs);
        const uint32_t p_addr = tc::smem_u32(recv);
        uint32_t n = 0, qr = 0, rows_done = 0;
        bool stop = false;
        auto pv = [&](uint32_t m, bool first) -> bool {
            if (!tc::mbar_wait(&bars->p_full, m & 1, abort_flag)) return false;
            if (first && !tc::mbar_wait(&bars->o_free, (rows_done & 1) ^ 1, abort_flag)) return false;
            tc::tc_fence_after();
            if (lane == 0) {
                const uint32_t v_addr = tc::smem_u32(stages + (m % kStages) * kStageBytes);
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    tc::mma_bf16(tmem_base + kTmemO, tc::sw128_desc(p_addr + kk * 32, 16, 1024),
                                 tc::sw128_desc(v_addr + kk * 2048, kKvBlk, 1024), kIdescPV,
                                 (first && kk == 0) ? 0u : 1u);
                tc::mma_commit(&bars->kv_empty[m % kStages]);
                tc::mma_commit_multicast(&bars->peer_free, (uint16_t)(1u << peer));
            }
            __syncwarp();
            return true;
        };
        for (int t = cluster; t < v.T_q && !stop; t += n_clusters) {
            const RowInfo r = load_row(v, t);
            const int32_t* idx_row = idx + (int64_t)t * K;
            const int ntiles = r.pos < 0 ? 0 : (int)ceil_div(row_extent(idx_row, K, lane), kBN);
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
                tc::tc_fence_after();
                if (lane == 0) {
                    const uint32_t kv_addr = tc::smem_u32(stages + st * kStageBytes);
                    const uint32_t d = tmem_base + kTmemS + sb * kBN;
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc::mma_bf16(d, tc::sw128_desc(q_addr + kb * kQBlk + kk * 32, 16, 1024),
                                         tc::sw128_desc(kv_addr + kb * kKvBlk + kk * 32, 16, 1024),
                                         kIdescQK, (kb | kk) ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        tc::mma_bf16(d, tc::sw64_desc(q_addr + 4 * kQBlk + kk * 32, 512),
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
    } else {
        // ---------------------------------------------------------------- softmax / exchange
        const int h = (warp & 3) * 32 + lane;          // head = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t my_recv = tc::smem_u32(recv) + h * (kBN * 4);
        const uint32_t peer_recv = tc::mapa_shared(my_recv, peer);
        const uint32_t peer_bar = tc::mapa_shared(tc::smem_u32(&bars->recv_full), peer);
        uint32_t n = 0, rows_done = 0;
        bool stop = false;
        for (int t = cluster; t < v.T_q && !stop; t += n_clusters) {
            const RowInfo r = load_row(v, t);
            const int32_t* idx_row = idx + (int64_t)t * K;
            const int ntiles = r.pos < 0 ? 0 : (int)ceil_div(row_extent(idx_row, K, lane), kBN);
            __nv_bfloat16* orow = out + ((int64_t)t * kH + h) * kDv + 256 * rank;
            if (ntiles == 0) {
                for (int c = 0; c < 256; c += 8)
                    *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
                if (lse != nullptr && rank == 0) lse[(int64_t)t * kH + h] = -INFINITY;
                continue;
            }
            float m_used = -INFINITY, l = 0.f;
            for (int j = 0; j < ntiles; ++j, ++n) {
                const uint32_t sb = n & 1;
                const int k0 = j * kBN;
                const uint32_t va = __ballot_sync(0xffffffffu, entry_valid(idx_row, K, k0 + lane, r.pos, v, warp == 2 && rank == 0));
                const uint32_t vb = __ballot_sync(0xffffffffu, entry_valid(idx_row, K, k0 + 32 + lane, r.pos, v, warp == 2 && rank == 0));
                if (!tc::mbar_wait(&bars->s_full[sb], (n >> 1) & 1, abort_flag)) {
                    stop = true;
                    break;
                }
                tc::tc_fence_after();
                float s[kBN];
                tc::tmem_ld32(tmem_base + lane_off + kTmemS + sb * kBN, s);
                tc::tmem_ld32(tmem_base + lane_off + kTmemS + sb * kBN + 32, s + 32);
                tc::tmem_ld_wait();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->s_empty[sb]);
                // swap partial S with the peer
                if (n > 0 && !tc::mbar_wait(&bars->peer_free, (n - 1) & 1, abort_flag)) {
                    stop = true;
                    break;
                }
                if (tid == 64) tc::mbar_arrive_expect_tx(&bars->recv_full, kRecvBytes);
#pragma unroll
                for (int i = 0; i < kBN / 4; ++i)
                    tc::st_async_v4(peer_recv + 16 * i, peer_bar, __float_as_uint(s[4 * i]),
                                    __float_as_uint(s[4 * i + 1]), __float_as_uint(s[4 * i + 2]),
                                    __float_as_uint(s[4 * i + 3]));
                if (!tc::mbar_wait_cluster(&bars->recv_full, n & 1, abort_flag)) {
                    stop = true;
                    break;
                }
                const float4* other = reinterpret_cast<const float4*>(recv + h * (kBN * 4));
#pragma unroll
                for (int i = 0; i < kBN / 4; ++i) {
                    const float4 o = other[i];
                    s[4 * i] += o.x;
                    s[4 * i + 1] += o.y;
                    s[4 * i + 2] += o.z;
                    s[4 * i + 3] += o.w;
                }
                tc::named_barrier(1, 128);  // every row of the buffer is read before P overwrites it
                // online softmax over the tile (base 2)
                float mt = -INFINITY;
#pragma unroll
                for (int i = 0; i < kBN; ++i) {
                    const bool ok = ((i < 32 ? va >> i : vb >> (i - 32)) & 1u) != 0;
                    s[i] = ok ? s[i] * scale_log2 : -INFINITY;
                    mt = fmaxf(mt, s[i]);
                }
                if (mt != -INFINITY) {
                    if (m_used == -INFINITY) {
                        m_used = mt;
                    } else if (mt > m_used + kRescaleLog2) {
                        // O of this head is final up to P.V(n-1) (receiving tile n implies it)
                        const float alpha = exp2f(m_used - mt);
                        m_used = mt;
                        l *= alpha;
#pragma unroll 1
                        for (int c = 0; c < 256; c += 32) {
                            float o[32];
                            tc::tmem_ld32(tmem_base + lane_off + kTmemO + c, o);
                            tc::tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 32; ++i) o[i] *= alpha;
                            tc::tmem_st32(tmem_base + lane_off + kTmemO + c, o);
                        }
                        tc::tmem_st_wait();
                    }
                }
                float psum = 0.f;
                uint32_t pk[kBN / 2];
#pragma unroll
                for (int i = 0; i < kBN; i += 2) {
                    const float p0 = s[i] == -INFINITY ? 0.f : exp2f(s[i] - m_used);
                    const float p1 = s[i + 1] == -INFINITY ? 0.f : exp2f(s[i + 1] - m_used);
                    psum += p0;
                    psum += p1;
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                    pk[i / 2] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                l += psum;
                // P row h, K-major 128-byte swizzle: 16-byte chunk c at (c ^ (h & 7))
                uint8_t* prow = recv + h * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4*>(prow + ((c ^ (h & 7)) * 16)) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                tc::fence_async_smem();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->p_full);
            }
            if (stop) break;
            // row epilogue: O / l -> bf16 -> global
            if (!tc::mbar_wait(&bars->o_ready, rows_done & 1, abort_flag)) break;
            tc::tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
            for (int c = 0; c < 256; c += 32) {
                float o[32];
                tc::tmem_ld32(tmem_base + lane_off + kTmemO + c, o);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                    uint32_t w4[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(o[i + 2 * q] * inv_l, o[i + 2 * q + 1] * inv_l);
                        w4[q] = *reinterpret_cast<const uint32_t*>(&b2);
                    }
                    *reinterpret_cast<uint4*>(orow + c + i) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->o_free);
            if (lse != nullptr && rank == 0)
                lse[(int64_t)t * kH + h] = l > 0.f ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
            ++rows_done;
        }
        // the peer's last P.V commit arrives here; take it before leaving
        if (!stop && n > 0) tc::mbar_wait(&bars->peer_free, (n - 1) & 1, abort_flag);
    }
    __syncwarp();
    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync_all();
    if (warp == 1) {
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
    if (a.q_dtype != HSA_BF16 || a.kv_dtype != HSA_BF16 || a.out_dtype != HSA_BF16) return false;
    if (a.H != kH || a.D_qk != kDqk || a.D_v != kDv) return false;
    auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    if (!al(a.q) || !al(a.kv) || !al(a.out)) return false;
    if ((uint64_t)a.seq.T_q * kH >= (1ull << 31)) return false;
    if ((uint64_t)a.seq.num_pages * a.seq.page_size >= (1ull << 31)) return false;
    return true;
}

size_t sparse_mla_tc_workspace(int32_t, int32_t) { return 0; }

cudaError_t launch_sparse_mla_tc(const SparseMlaArgs& a, cudaStream_t st) {
    if (a.seq.T_q == 0) return cudaSuccess;
    const uint64_t slots = (uint64_t)a.seq.num_pages * a.seq.page_size;
    const uint64_t qrows = (uint64_t)a.seq.T_q * kH;
    CUtensorMap tql, tqr, tkl, tkr;
    bool ok = make_tensor_map_2d(&tql, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qrows, kDqk, kDqk * 2,
                                 64, kH, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_tensor_map_2d(&tqr, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qrows, kDqk, kDqk * 2,
                                 32, kH, CU_TENSOR_MAP_SWIZZLE_64B) &&
              make_tensor_map_2d(&tkl, a.kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, slots, kDqk, kDqk * 2,
                                 64, 1, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_tensor_map_2d(&tkr, a.kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, slots, kDqk, kDqk * 2,
                                 32, 1, CU_TENSOR_MAP_SWIZZLE_64B);
    if (!ok) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(sparse_mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmem);
    if (e != cudaSuccess) return e;
    const int clusters = std::max(1, std::min(a.seq.T_q, num_sms() / 2));
    const float scale_log2 = a.softmax_scale * 1.4426950408889634f;
    sparse_mla_tc_kernel<<<2 * clusters, kThreads, kSmem, st>>>(
        tql, tqr, tkl, tkr, a.seq, a.idx, a.K, scale_log2, reinterpret_cast<__nv_bfloat16*>(a.out), a.lse);
    count_launch();
    return cudaGetLastError();
}

}  // namespace hsa
