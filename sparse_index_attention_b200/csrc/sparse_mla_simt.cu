// sparse_mla_simt.cu -- CUDA-core sparse MLA attention for any head count and latent width.
//
// "Day-One Inference Adaptation for Very Large Hybrid-Attention Models", 3.2: partition by
// query, aggregate over the selected positions, stage them in shared memory.  A CTA owns one
// query row and kHeads heads; it walks the row's selected positions in tiles of kRows, gathers
// each selected cache row through the block table into shared memory (latent || rope, widened
// to fp32; FP8 latent codes are decoded and multiplied by the per-token scale), and keeps an
// online softmax (running max, running sum, rescaled fp32 accumulator) per head.
#include "kernels.h"

namespace hsa {

namespace {

constexpr int kThreads = 256;
constexpr int kHeads = 8;
constexpr int kRows = 32;  // kHeads * kRows == kThreads: one logit per thread per tile

template <typename QT, int KVT, typename OT>  // KVT: 0 fp32 packed, 1 bf16 packed, 2 e4m3 + bf16 rope
__global__ void __launch_bounds__(kThreads)
sparse_mla_simt_kernel(SeqView v, const QT* __restrict__ q, int H, int D_qk, int D_v,
                       const void* __restrict__ kv, const float* __restrict__ kv_scale, int kv_group,
                       const __nv_bfloat16* __restrict__ kv_rope, const int32_t* __restrict__ idx,
                       int K, float softmax_scale, OT* __restrict__ out, float* __restrict__ lse) {
    extern __shared__ float smem[];
    float* sq = smem;                          // [kHeads, D_qk]
    float* skv = sq + kHeads * D_qk;           // [kRows, D_qk]
    float* so = skv + kRows * D_qk;            // [kHeads, D_v]
    float* sz = so + kHeads * D_v;             // [kHeads, kRows] logits, then probabilities
    float* sm_ = sz + kHeads * kRows;          // [kHeads] running max
    float* sl = sm_ + kHeads;                  // [kHeads] running sum
    float* salpha = sl + kHeads;               // [kHeads] rescale of this tile
    __shared__ long long sslot[kRows];         // physical slot of each tile row (-1: none)

    const int t = blockIdx.x;
    const int h0 = blockIdx.y * kHeads;
    const int nh = min(kHeads, H - h0);
    const RowInfo r = load_row(v, t);
    const int tid = threadIdx.x;
    const int D_rope = D_qk - D_v;

    for (int i = tid; i < kHeads * D_qk; i += kThreads) {
        const int h = i / D_qk, d = i % D_qk;
        sq[i] = h < nh ? to_f32(q[((int64_t)t * H + h0 + h) * D_qk + d]) : 0.f;
    }
    for (int i = tid; i < kHeads * D_v; i += kThreads) so[i] = 0.f;
    if (tid < kHeads) {
        sm_[tid] = -INFINITY;
        sl[tid] = 0.f;
    }
    __syncthreads();

    const int32_t* sel = idx + (int64_t)t * K;
    for (int k0 = 0; k0 < K && r.pos >= 0; k0 += kRows) {
        if (tid < kRows) {
            long long s64 = -1;
            if (k0 + tid < K) {
                const int n = sel[k0 + tid];
                if (n != -1) {
                    if (n < 0 || n > r.pos)
                        flag_status(v, HSA_DEV_BAD_POS);
                    else
                        s64 = paged_slot(v, r.b, n);
                }
            }
            sslot[tid] = s64;
        }
        __syncthreads();
        // gather the tile's rows into shared memory as fp32
        for (int i = tid; i < kRows * D_qk; i += kThreads) {
            const int rr = i / D_qk, d = i % D_qk;
            float x = 0.f;
            if (sslot[rr] >= 0) {
                const int64_t s = sslot[rr];
                if (KVT == 0) {
                    x = reinterpret_cast<const float*>(kv)[s * D_qk + d];
                } else if (KVT == 1) {
                    x = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(kv)[s * D_qk + d]);
                } else {
                    x = d < D_v ? e4m3_to_f32(reinterpret_cast<const uint8_t*>(kv)[s * D_v + d]) *
                                      kv_scale[s * (D_v / kv_group) + d / kv_group]
                                : __bfloat162float(kv_rope[s * D_rope + (d - D_v)]);
                }
            }
            skv[i] = x;
        }
        __syncthreads();
        {   // logits: thread (h, rr)
            const int h = tid / kRows, rr = tid % kRows;
            float z = -INFINITY;
            if (sslot[rr] >= 0 && h < nh) {
                float dot = 0.f;
                const float* qh = sq + h * D_qk;
                const float* kr = skv + rr * D_qk;
                for (int d = 0; d < D_qk; ++d) dot = fmaf(qh[d], kr[d], dot);
                z = dot * softmax_scale;
            }
            sz[h * kRows + rr] = z;
        }
        __syncthreads();
        if (tid < kHeads) {  // online softmax bookkeeping per head
            const int h = tid;
            float mt = -INFINITY;
            for (int rr = 0; rr < kRows; ++rr) mt = fmaxf(mt, sz[h * kRows + rr]);
            const float m_old = sm_[h];
            const float m_new = fmaxf(m_old, mt);
            float alpha = 1.f, sum = 0.f;
            if (m_new != -INFINITY) {
                alpha = m_old == -INFINITY ? 0.f : expf(m_old - m_new);
                for (int rr = 0; rr < kRows; ++rr) {
                    const float z = sz[h * kRows + rr];
                    const float p = z == -INFINITY ? 0.f : expf(z - m_new);
                    sz[h * kRows + rr] = p;
                    sum += p;
                }
            } else {
                for (int rr = 0; rr < kRows; ++rr) sz[h * kRows + rr] = 0.f;
            }
            sm_[h] = m_new;
            sl[h] = sl[h] * alpha + sum;
            salpha[h] = alpha;
        }
        __syncthreads();
        for (int i = tid; i < kHeads * D_v; i += kThreads) {
            const int h = i / D_v, d = i % D_v;
            float acc = so[i] * salpha[h];
            const float* p = sz + h * kRows;
            for (int rr = 0; rr < kRows; ++rr) acc = fmaf(p[rr], skv[rr * D_qk + d], acc);
            so[i] = acc;
        }
        __syncthreads();
    }
    for (int i = tid; i < nh * D_v; i += kThreads) {
        const int h = i / D_v, d = i % D_v;
        const float l = sl[h];
        const float o = l > 0.f ? so[i] / l : 0.f;
        const int64_t off = ((int64_t)t * H + h0 + h) * D_v + d;
        if constexpr (sizeof(OT) == 4) out[off] = o;
        else out[off] = __float2bfloat16(o);
    }
    if (lse != nullptr && tid < nh) {
        const float l = sl[tid];
        lse[(int64_t)t * H + h0 + tid] = l > 0.f ? sm_[tid] + logf(l) : -INFINITY;
    }
}

template <typename QT, int KVT, typename OT>
cudaError_t launch_t(const SparseMlaArgs& a, cudaStream_t st) {
    dim3 grid((unsigned)a.seq.T_q, (unsigned)ceil_div(a.H, kHeads));
    size_t smem = sizeof(float) * ((size_t)kHeads * a.D_qk + (size_t)kRows * a.D_qk +
                                   (size_t)kHeads * a.D_v + kHeads * kRows + 3 * kHeads);
    auto k = sparse_mla_simt_kernel<QT, KVT, OT>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, smem, st>>>(a.seq, reinterpret_cast<const QT*>(a.q), a.H, a.D_qk, a.D_v,
                                    a.kv, a.kv_scale, a.kv_scale_group,
                                    reinterpret_cast<const __nv_bfloat16*>(a.kv_rope), a.idx, a.K,
                                    a.softmax_scale, reinterpret_cast<OT*>(a.out), a.lse);
    count_launch();
    return cudaGetLastError();
}

template <typename QT, typename OT>
cudaError_t launch_q(const SparseMlaArgs& a, cudaStream_t st) {
    if (a.kv_dtype == HSA_F32) return launch_t<QT, 0, OT>(a, st);
    if (a.kv_dtype == HSA_BF16) return launch_t<QT, 1, OT>(a, st);
    return launch_t<QT, 2, OT>(a, st);
}

}  // namespace

cudaError_t launch_sparse_mla_simt(const SparseMlaArgs& a, cudaStream_t st) {
    if (a.seq.T_q == 0) return cudaSuccess;
    if (a.q_dtype == HSA_F32) {
        return a.out_dtype == HSA_F32 ? launch_q<float, float>(a, st)
                                      : launch_q<float, __nv_bfloat16>(a, st);
    }
    return a.out_dtype == HSA_F32 ? launch_q<__nv_bfloat16, float>(a, st)
                                  : launch_q<__nv_bfloat16, __nv_bfloat16>(a, st);
}

}  // namespace hsa
