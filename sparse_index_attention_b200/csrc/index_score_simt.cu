// index_score_simt.cu -- CUDA-core index score for any (H_I, D_I) and storage type.
//
// One thread per (query row, history position): the thread walks the key row of its position
// once per index head, keeps the dot product in fp32 and folds it into the head-weighted ReLU
// sum (the relevance score of "Day 0 Inference Adaptation and Optimization for Hybrid Attention
// Models", "Sparse Attention Pipeline Optimization").  Serves the fp32 workloads and shapes the
// tensor-core kernel does not take.
#include "kernels.h"

namespace hsa {

namespace {

constexpr int kThreads = 128;

// KT: 0 fp32 keys, 1 bf16 keys, 2 e4m3 keys + per-key fp32 scale, 3 MXFP8 keys (e4m3 codes,
// one E8M0 byte per 32 dims, applied to each element: the scale varies along the dot product).
// QT = uint8_t: MXFP8 queries (codes, q_scale one E8M0 byte per 32 dims), decoded on load.
template <typename QT, int KT>
__global__ void __launch_bounds__(kThreads)
index_score_simt_kernel(SeqView v, const QT* __restrict__ q_I, const uint8_t* __restrict__ q_scale,
                        const float* __restrict__ w,
                        int H_I, int D_I, const void* __restrict__ k_cache,
                        const void* __restrict__ k_scale, float* __restrict__ scores, int64_t ld) {
    extern __shared__ float smem[];
    float* sq = smem;                 // [H_I * D_I]
    float* sw = smem + H_I * D_I;     // [H_I]
    const int t = blockIdx.y;
    const RowInfo r = load_row(v, t);
    const int s0 = blockIdx.x * kThreads;
    if (r.pos < 0 || s0 > r.pos) return;  // uniform over the block
    const int64_t qoff = (int64_t)t * H_I * D_I;
    for (int i = threadIdx.x; i < H_I * D_I; i += kThreads) {
        if constexpr (sizeof(QT) == 1)
            sq[i] = e4m3_to_f32(q_I[qoff + i]) * e8m0_to_f32(q_scale[(qoff + i) / 32]);
        else
            sq[i] = to_f32(q_I[qoff + i]);
    }
    for (int i = threadIdx.x; i < H_I; i += kThreads) sw[i] = w[(int64_t)t * H_I + i];
    __syncthreads();
    const int s = s0 + threadIdx.x;
    if (s > r.pos) return;
    const int64_t slot = paged_slot(v, r.b, s);
    float acc = 0.f;
    for (int j = 0; j < H_I; ++j) {
        float dot = 0.f;
        const float* qj = sq + j * D_I;
        for (int d = 0; d < D_I; ++d) {
            float kd;
            if (KT == 0)
                kd = reinterpret_cast<const float*>(k_cache)[slot * D_I + d];
            else if (KT == 1)
                kd = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(k_cache)[slot * D_I + d]);
            else if (KT == 2)
                kd = e4m3_to_f32(reinterpret_cast<const uint8_t*>(k_cache)[slot * D_I + d]);
            else
                kd = e4m3_to_f32(reinterpret_cast<const uint8_t*>(k_cache)[slot * D_I + d]) *
                     e8m0_to_f32(reinterpret_cast<const uint8_t*>(k_scale)[slot * (D_I / 32) + d / 32]);
            dot = fmaf(qj[d], kd, dot);
        }
        acc = fmaf(sw[j], fmaxf(dot, 0.f), acc);
    }
    if (KT == 2) acc *= reinterpret_cast<const float*>(k_scale)[slot];  // positive per-key scale
                                                                        // factors out of the ReLU sum
    scores[(int64_t)t * ld + s] = acc;
}

template <typename QT, int KT>
cudaError_t launch_t(const IndexScoreArgs& a, cudaStream_t st) {
    dim3 grid((unsigned)ceil_div(a.max_seq_len, kThreads), (unsigned)a.seq.T_q);
    size_t smem = sizeof(float) * ((size_t)a.H_I * a.D_I + a.H_I);
    auto k = index_score_simt_kernel<QT, KT>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k<<<grid, kThreads, smem, st>>>(a.seq, reinterpret_cast<const QT*>(a.q_I),
                                    static_cast<const uint8_t*>(a.q_scale), a.w, a.H_I, a.D_I,
                                    a.k_cache, a.k_scale, a.scores, a.ld);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_index_score_simt(const IndexScoreArgs& a, cudaStream_t st) {
    if (a.q_dtype == HSA_MXE4M3) return launch_t<uint8_t, 3>(a, st);   // MX queries need MX keys
    if (a.q_dtype == HSA_F32) {
        if (a.k_dtype == HSA_F32) return launch_t<float, 0>(a, st);
        if (a.k_dtype == HSA_BF16) return launch_t<float, 1>(a, st);
        if (a.k_dtype == HSA_MXE4M3) return launch_t<float, 3>(a, st);
        return launch_t<float, 2>(a, st);
    }
    if (a.k_dtype == HSA_F32) return launch_t<__nv_bfloat16, 0>(a, st);
    if (a.k_dtype == HSA_BF16) return launch_t<__nv_bfloat16, 1>(a, st);
    if (a.k_dtype == HSA_MXE4M3) return launch_t<__nv_bfloat16, 3>(a, st);
    return launch_t<__nv_bfloat16, 2>(a, st);
}

}  // namespace hsa
