// Log-sum-exp weighted reduction of the partial results of one decode step.
//
// "ZoRRo Inference & Forest Cascade Attention", "Core Mechanism" step 3:
// the grouped (prefix) and per-request (suffix) partial results are reduced
// with their log-sum-exp weights.  For each (request r, query head hq) the
// partials are, in order, every split chunk of every group on r's chain and
// every split chunk of r's own pass:
//     lse = log(sum_i exp(lse_i)),   out = sum_i exp(lse_i - lse) * o_i,
// with o_i already normalised by its own softmax sum.  One warp per
// (r, hq).  The partials are taken 32 at a time: lane i finds the row of
// partial i of the batch and reads its lse, one shuffle reduction gives the
// batch maximum and weight sum (the running state is rescaled when the
// maximum grows), then the o rows stream in four at a time, each lane owning
// a contiguous slice of head_dim.  Partials with lse = -inf (empty chunks)
// are skipped without reading their rows.
#include <cuda_bf16.h>

#include "fca_internal.h"

namespace fca {

struct MergeArgs {
    int32_t R, Hq, G;
    const int32_t* chain_off;
    const int32_t* chain_g;
    const int32_t* chain_pos;
    const int32_t* g_nch;
    const int32_t* g_nm;
    const int32_t* g_part;
    const int32_t* s_nch;
    const int32_t* s_part;
    const float* part_o;
    const float* part_lse;
    __nv_bfloat16* out;
    float* lse;
};

namespace {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int V>
__device__ __forceinline__ void load_row(const float* src, float (&o)[V]) {
    if constexpr (V == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(src));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    } else {
        const float2 v = __ldg(reinterpret_cast<const float2*>(src));
        o[0] = v.x; o[1] = v.y;
    }
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(256) k_merge(MergeArgs a) {
    constexpr int V = D / 32;   // floats per lane
    constexpr int kInFlight = 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t pair = (int64_t)blockIdx.x * 8 + warp;
    if (pair >= (int64_t)a.R * a.Hq) return;
    const int32_t r = (int32_t)(pair / a.Hq), hq = (int32_t)(pair % a.Hq);
    const int32_t h = hq / a.G, gq = hq % a.G;
    const int32_t c0 = a.chain_off[r], c1 = a.chain_off[r + 1];
    const int32_t nsc = a.s_nch[r];
    int32_t n = nsc;
    for (int32_t c = c0; c < c1; ++c) n += a.g_nch[a.chain_g[c]];

    // row of partial k of this pair (-1 past the end)
    auto partial_row = [&](int32_t k) -> int32_t {
        for (int32_t c = c0; c < c1; ++c) {
            const int32_t g = a.chain_g[c], nch = a.g_nch[g];
            if (k < nch) return a.g_part[g] + ((h * nch + k) * a.g_nm[g] + a.chain_pos[c]) * a.G + gq;
            k -= nch;
        }
        return k < nsc ? a.s_part[r] + (h * nsc + k) * a.G + gq : -1;
    };

    float m = -INFINITY, l = 0.f;
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;

    for (int32_t b0 = 0; b0 < n; b0 += 32) {
        const int32_t row = partial_row(b0 + lane);
        const float li = row >= 0 ? __ldg(a.part_lse + row) : -INFINITY;
        const float mb = warp_max(li);
        if (mb == -INFINITY) continue;              // every partial of the batch is empty
        const float m_new = fmaxf(m, mb);
        const float sc = expf(m - m_new);           // 0 while nothing has been added
        l *= sc;
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] *= sc;
        const float wi = li == -INFINITY ? 0.f : expf(li - m_new);
        l += warp_sum(wi);
        m = m_new;
        const int32_t nb = min(32, n - b0);
        for (int32_t j0 = 0; j0 < nb; j0 += kInFlight) {
            float o[kInFlight][V], w[kInFlight];
#pragma unroll
            for (int u = 0; u < kInFlight; ++u) {
                const int32_t j = j0 + u;
                const int32_t rj = __shfl_sync(0xffffffffu, row, j & 31);
                w[u] = __shfl_sync(0xffffffffu, wi, j & 31);
                if (j >= nb) w[u] = 0.f;
                if (w[u] > 0.f) {
                    load_row<V>(a.part_o + (int64_t)rj * D + lane * V, o[u]);
                } else {
#pragma unroll
                    for (int i = 0; i < V; ++i) o[u][i] = 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < kInFlight; ++u)
#pragma unroll
                for (int i = 0; i < V; ++i) acc[i] = fmaf(w[u], o[u][i], acc[i]);
        }
    }

    const float inv = l > 0.f ? 1.f / l : 0.f;
    __nv_bfloat16* dst = a.out + pair * D + lane * V;
#pragma unroll
    for (int i = 0; i < V; i += 2) {
        *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(acc[i] * inv, acc[i + 1] * inv);
    }
    if (a.lse && lane == 0) a.lse[pair] = l > 0.f ? m + logf(l) : -INFINITY;
}

cudaError_t launch_merge(const fca_plan_s* P, void* out, float* lse, cudaStream_t stream) {
    MergeArgs a;
    a.R = P->R;
    a.Hq = P->Hq;
    a.G = P->G;
    a.chain_off = P->chain_off;
    a.chain_g = P->chain_g;
    a.chain_pos = P->chain_pos;
    a.g_nch = P->g_nch;
    a.g_nm = P->g_nm;
    a.g_part = P->g_part;
    a.s_nch = P->s_nch;
    a.s_part = P->s_part;
    a.part_o = P->part_o;
    a.part_lse = P->part_lse;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.lse = lse;
    const int64_t pairs = (int64_t)P->R * P->Hq;
    const int grid = (int)((pairs + 7) / 8);
    if (P->D == 128)
        k_merge<128><<<grid, 256, 0, stream>>>(a);
    else
        k_merge<64><<<grid, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace fca
