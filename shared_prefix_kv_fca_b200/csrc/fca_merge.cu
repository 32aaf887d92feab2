// Log-sum-exp weighted reduction of the partial results of one decode step.
//
// "ZoRRo Inference & Forest Cascade Attention", "Core Mechanism" step 3:
// the grouped (prefix) and per-request (suffix) partial results are reduced
// with their log-sum-exp weights.  For each (request r, query head hq) the
// partials are, in order, every split chunk of every group on r's chain and
// every split chunk of r's own pass:
//     lse = log(sum_i exp(lse_i)),   out = sum_i exp(lse_i - lse) * o_i,
// with o_i already normalised by its own softmax sum.  One warp per
// (r, hq); lanes own contiguous slices of head_dim; a single online pass with
// max-rescaling, so each partial row is read once.
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

template <int D>
__global__ void __launch_bounds__(256) k_merge(MergeArgs a) {
    constexpr int V = D / 32;   // floats per lane
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t pair = (int64_t)blockIdx.x * 8 + warp;
    if (pair >= (int64_t)a.R * a.Hq) return;
    const int32_t r = (int32_t)(pair / a.Hq), hq = (int32_t)(pair % a.Hq);
    const int32_t h = hq / a.G, gq = hq % a.G;

    float m = -INFINITY, l = 0.f;
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;

    auto add = [&](int32_t p) {
        const float li = __ldg(a.part_lse + p);
        if (li == -INFINITY) return;
        float o[V];
        const float* src = a.part_o + (int64_t)p * D + lane * V;
        if constexpr (V == 4) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(src));
            o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
        } else {
            const float2 v = __ldg(reinterpret_cast<const float2*>(src));
            o[0] = v.x; o[1] = v.y;
        }
        if (li > m) {
            const float sc = expf(m - li);
            l *= sc;
#pragma unroll
            for (int i = 0; i < V; ++i) acc[i] *= sc;
            m = li;
        }
        const float w = expf(li - m);
        l += w;
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = fmaf(w, o[i], acc[i]);
    };

    for (int32_t c = a.chain_off[r]; c < a.chain_off[r + 1]; ++c) {
        const int32_t g = a.chain_g[c], pos = a.chain_pos[c];
        const int32_t nch = a.g_nch[g], nm = a.g_nm[g], base = a.g_part[g];
        for (int32_t ch = 0; ch < nch; ++ch) add(base + ((h * nch + ch) * nm + pos) * a.G + gq);
    }
    const int32_t nsc = a.s_nch[r];
    for (int32_t ch = 0; ch < nsc; ++ch) add(a.s_part[r] + (h * nsc + ch) * a.G + gq);

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
