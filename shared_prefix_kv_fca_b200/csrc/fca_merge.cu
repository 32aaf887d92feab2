// Log-sum-exp weighted reduction of the partial results of one decode step.
//
// "ZoRRo Inference & Forest Cascade Attention", "Core Mechanism" step 3:
// the grouped (prefix) and per-request (suffix) partial results are reduced
// with their log-sum-exp weights.  For each (request r, query head hq) the
// partials are, in order, every split chunk of every group on r's chain and
// every split chunk of r's own pass:
//     lse = log(sum_i exp(lse_i)),   out = sum_i exp(lse_i - lse) * o_i,
// with o_i already normalised by its own softmax sum.
//
// Work unit: (request, KV head, slab of up to four of that KV head's query
// heads), taken by W warps (W = 1, 2, 4 or 8, more when there are few units
// and many partials per unit).  Every pass writes the G query heads of one
// (request, KV head, chunk) as G consecutive partial rows, so a slab's rows of
// one partial are one contiguous run of 4 x head_dim floats: each lane owns
// float4 slots of that run, and the request's group chain is walked once per
// slab, not once per query head.  The chain entries are read by one lane each
// (all in parallel) and a warp scan turns their chunk counts into partial
// offsets, so locating partial k costs shuffles rather than dependent loads.
//
// Warp w of a unit takes partials w, w + W, w + 2W, ... 32 at a time: lane i
// locates partial i of the batch and reads its lse values; shuffle reductions
// give each head's batch maximum and weight sum (the running state is
// rescaled when a maximum grows); then the rows are accumulated two partials
// at a time.  Partials with lse = -inf (empty chunks) never contribute.  With
// W > 1 the warps' states (maximum, sum, accumulator) are combined through
// shared memory.  A unit's warps share one CTA, so W > 1 only when units are
// few (about 8 warps per SM in all) and each has many partials to read.
#include <cuda_bf16.h>

#include "fca_device.cuh"
#include "fca_internal.h"

namespace fca {

struct MergeArgs {
    int32_t R, Hq, Hkv, G, n_slabs, W;
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
    const int32_t* m_ng;      // null: walk the chain
    const int2* m_rec;
};

namespace {

constexpr int kSlabHeads = 4;   // query heads per unit
constexpr int kWarps = 8;       // warps per CTA
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

__device__ __forceinline__ int32_t warp_incl_scan(int32_t v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// a[i] for a lane-dependent i, without indexing a register array at run time
__device__ __forceinline__ float pick(const float (&a)[kSlabHeads], int i) {
    float r = a[0];
#pragma unroll
    for (int k = 1; k < kSlabHeads; ++k) r = (i == k) ? a[k] : r;
    return r;
}

template <int D>
struct MergeSmem {
    static constexpr int kSlots = kSlabHeads * D / 128;
    float4 acc[kWarps][kSlots][32];
    float m[kWarps][kSlabHeads];
    float l[kWarps][kSlabHeads];
};

}  // namespace

template <int D>
__global__ void __launch_bounds__(256, 3) k_merge(MergeArgs a) {
    constexpr int kSlots = kSlabHeads * D / 128;   // float4 slots per lane
    constexpr int kInFlight = 2;                    // partials loaded together
    __shared__ MergeSmem<D> sm;
    // launched after a pass with programmatic serialization: its rows are
    // complete and visible past this point
    dev::pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = a.W, sub = warp % W;
    const int64_t unit = (int64_t)blockIdx.x * (kWarps / W) + warp / W;
    const bool active = unit < (int64_t)a.R * a.Hkv * a.n_slabs;   // uniform across a unit's warps
    const int32_t slab = active ? (int32_t)(unit % a.n_slabs) : 0;
    const int32_t rh = active ? (int32_t)(unit / a.n_slabs) : 0;
    const int32_t r = rh / a.Hkv, h = rh % a.Hkv;
    const int32_t gq0 = slab * kSlabHeads;
    const int32_t nh = min(kSlabHeads, a.G - gq0);   // valid heads of this slab

    // slot j of this lane: float index f = j * 128 + lane * 4 of the slab's run
    int slot_head[kSlots];
#pragma unroll
    for (int j = 0; j < kSlots; ++j) slot_head[j] = (j * 128 + lane * 4) / D;

    float m[kSlabHeads], l[kSlabHeads];
#pragma unroll
    for (int i = 0; i < kSlabHeads; ++i) { m[i] = -INFINITY; l[i] = 0.f; }
    float4 acc[kSlots];
#pragma unroll
    for (int j = 0; j < kSlots; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);

    if (active) {
        // ---- the request's partials: chain entries (one lane each), then its own chunks
        const int32_t nsc = a.s_nch[r], spart = a.s_part[r];
        // The planner's record of the group partials (one entry each, read
        // with the request's own counts, no dependent loads) when it holds
        // them all; else the chain walk.
        const int32_t ng = a.m_ng ? a.m_ng[r] : kMergeRec + 1;
        // (read whatever the count is, so that it does not wait for the count)
        const int2 rec = (a.m_rec && lane < kMergeRec) ? a.m_rec[(int64_t)r * kMergeRec + lane] : make_int2(0, 0);
        const bool recorded = ng <= kMergeRec;
        const int32_t c0 = recorded ? 0 : a.chain_off[r];
        const int32_t depth = recorded ? ng : a.chain_off[r + 1] - c0;
        const bool wide = depth < 32;   // warp-uniform: every entry fits one lane
        int32_t e_nch = 0, e_base = 0, e_step = 0;
        if (recorded) {
            if (lane < depth) {
                e_nch = 1;
                e_base = rec.x + h * rec.y + gq0;
            } else if (lane == depth) {
                e_nch = nsc;
                e_base = spart + h * nsc * a.G + gq0;
                e_step = a.G;
            }
        } else if (wide) {
            // entry e < depth: group chain[e]; row of (chunk k, slab) =
            //   g_part + ((h nch + k) nm + pos) G + gq0 = e_base + k * e_step
            // entry depth: own chunks, row = s_part + (h nsc + k) G + gq0
            if (lane < depth) {
                const int32_t g = a.chain_g[c0 + lane], pos = a.chain_pos[c0 + lane];
                const int32_t nch = a.g_nch[g], nm = a.g_nm[g];
                e_nch = nch;
                e_base = a.g_part[g] + ((h * nch) * nm + pos) * a.G + gq0;
                e_step = nm * a.G;
            } else if (lane == depth) {
                e_nch = nsc;
                e_base = spart + h * nsc * a.G + gq0;
                e_step = a.G;
            }
        }
        const int32_t e_end = warp_incl_scan(e_nch, lane);   // exclusive end of entry's partials
        int32_t n = nsc;
        if (wide) {
            n = __shfl_sync(kFull, e_end, depth);
        } else {   // (never for a recorded request: depth <= kMergeRec)
            for (int32_t c = c0; c < c0 + depth; ++c) n += a.g_nch[a.chain_g[c]];
        }

        const int32_t n_mine = n > sub ? (n - sub + W - 1) / W : 0;   // partials sub, sub + W, ...
        for (int32_t b0 = 0; b0 < n_mine; b0 += 32) {
            // row of the slab's first head in partial k of the request (-1 past the end)
            int32_t row = -1;
            int32_t k = (b0 + lane) * W + sub;
            if (wide) {
                int32_t e = 0;
                for (int32_t i = 0; i < depth; ++i) e += (k >= __shfl_sync(kFull, e_end, i)) ? 1 : 0;
                const int32_t end = __shfl_sync(kFull, e_end, e);
                const int32_t cnt = __shfl_sync(kFull, e_nch, e);
                const int32_t base = __shfl_sync(kFull, e_base, e);
                const int32_t step = __shfl_sync(kFull, e_step, e);
                if (k < n) row = base + (k - (end - cnt)) * step;
            } else if (k < n) {
                for (int32_t c = c0; c < c0 + depth && row < 0; ++c) {
                    const int32_t g = a.chain_g[c], nch = a.g_nch[g];
                    if (k < nch) row = a.g_part[g] + ((h * nch + k) * a.g_nm[g] + a.chain_pos[c]) * a.G + gq0;
                    k -= nch;
                }
                if (row < 0) row = spart + (h * nsc + k) * a.G + gq0;
            }
            float li[kSlabHeads], wi[kSlabHeads], sc[kSlabHeads];
#pragma unroll
            for (int i = 0; i < kSlabHeads; ++i)
                li[i] = (row >= 0 && i < nh) ? __ldg(a.part_lse + row + i) : -INFINITY;
#pragma unroll
            for (int i = 0; i < kSlabHeads; ++i) {
                const float m_new = fmaxf(m[i], warp_max(li[i]));
                sc[i] = m_new == -INFINITY ? 1.f : expf(m[i] - m_new);   // 0 while nothing has been added
                wi[i] = li[i] == -INFINITY ? 0.f : expf(li[i] - m_new);
                l[i] = l[i] * sc[i] + warp_sum(wi[i]);
                m[i] = m_new;
            }
#pragma unroll
            for (int j = 0; j < kSlots; ++j) {
                const float s = pick(sc, slot_head[j]);
                acc[j].x *= s; acc[j].y *= s; acc[j].z *= s; acc[j].w *= s;
            }
            const int32_t nb = min(32, n_mine - b0);
            for (int32_t j0 = 0; j0 < nb; j0 += kInFlight) {
                float4 o[kInFlight][kSlots];
                float w[kInFlight][kSlots];
#pragma unroll
                for (int u = 0; u < kInFlight; ++u) {
                    const int32_t jj = (j0 + u) & 31;
                    const int32_t rj = __shfl_sync(kFull, row, jj);
                    float wh[kSlabHeads];
#pragma unroll
                    for (int i = 0; i < kSlabHeads; ++i) wh[i] = __shfl_sync(kFull, wi[i], jj);
                    const float* src = a.part_o + (int64_t)rj * D + lane * 4;
#pragma unroll
                    for (int j = 0; j < kSlots; ++j) {
                        w[u][j] = (j0 + u < nb && slot_head[j] < nh) ? pick(wh, slot_head[j]) : 0.f;
                        o[u][j] = w[u][j] > 0.f ? __ldg(reinterpret_cast<const float4*>(src + j * 128))
                                                : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
#pragma unroll
                for (int u = 0; u < kInFlight; ++u)
#pragma unroll
                    for (int j = 0; j < kSlots; ++j) {
                        acc[j].x = fmaf(w[u][j], o[u][j].x, acc[j].x);
                        acc[j].y = fmaf(w[u][j], o[u][j].y, acc[j].y);
                        acc[j].z = fmaf(w[u][j], o[u][j].z, acc[j].z);
                        acc[j].w = fmaf(w[u][j], o[u][j].w, acc[j].w);
                    }
            }
        }
    }

    // ---- combine the W warps of a unit (W is uniform across the CTA)
    if (W > 1) {
#pragma unroll
        for (int j = 0; j < kSlots; ++j) sm.acc[warp][j][lane] = acc[j];
        if (lane < kSlabHeads) {
            sm.m[warp][lane] = pick(m, lane);
            sm.l[warp][lane] = pick(l, lane);
        }
        __syncthreads();
        if (sub != 0) return;
#pragma unroll
        for (int i = 0; i < kSlabHeads; ++i) {
            float mm = -INFINITY;
            for (int v = 0; v < W; ++v) mm = fmaxf(mm, sm.m[warp + v][i]);
            float ll = 0.f;
            for (int v = 0; v < W; ++v) {
                const float mv = sm.m[warp + v][i];
                ll += mv == -INFINITY ? 0.f : sm.l[warp + v][i] * expf(mv - mm);
            }
            m[i] = mm;
            l[i] = ll;
        }
#pragma unroll
        for (int j = 0; j < kSlots; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int v = 0; v < W; ++v) {
            float f[kSlabHeads];
#pragma unroll
            for (int i = 0; i < kSlabHeads; ++i) {
                const float mv = sm.m[warp + v][i];
                f[i] = mv == -INFINITY ? 0.f : expf(mv - m[i]);
            }
#pragma unroll
            for (int j = 0; j < kSlots; ++j) {
                const float s = pick(f, slot_head[j]);
                const float4 x = sm.acc[warp + v][j][lane];
                acc[j].x = fmaf(s, x.x, acc[j].x);
                acc[j].y = fmaf(s, x.y, acc[j].y);
                acc[j].z = fmaf(s, x.z, acc[j].z);
                acc[j].w = fmaf(s, x.w, acc[j].w);
            }
        }
    }
    if (!active) return;

    // ---- normalise and store: out[r][h G + gq0 + head][col], lse[r][h G + gq0 + head]
    float inv[kSlabHeads];
#pragma unroll
    for (int i = 0; i < kSlabHeads; ++i) inv[i] = l[i] > 0.f ? 1.f / l[i] : 0.f;
    const int64_t q0 = (int64_t)r * a.Hq + (int64_t)h * a.G + gq0;   // first query head of the slab
#pragma unroll
    for (int j = 0; j < kSlots; ++j) {
        if (slot_head[j] >= nh) continue;
        const float s = pick(inv, slot_head[j]);
        uint2 v;
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc[j].x * s, acc[j].y * s);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc[j].z * s, acc[j].w * s);
        v.x = *reinterpret_cast<uint32_t*>(&lo);
        v.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(a.out + q0 * D + j * 128 + lane * 4) = v;
    }
    if (a.lse && lane < nh) {
        const float mm = pick(m, lane), ll = pick(l, lane);
        a.lse[q0 + lane] = ll > 0.f ? mm + logf(ll) : -INFINITY;
    }
}

// after_pass: launched right behind the pass that ends the step on the same
// stream, with programmatic serialization, so that the grid is set up while
// that pass runs out (its CTAs wait for it before reading a partial row).
cudaError_t launch_merge(const fca_plan_s* P, void* out, float* lse, bool after_pass, cudaStream_t stream) {
    MergeArgs a;
    a.R = P->R;
    a.Hq = P->Hq;
    a.Hkv = P->Hkv;
    a.G = P->G;
    a.n_slabs = (P->G + kSlabHeads - 1) / kSlabHeads;
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
    a.m_ng = P->m_ng;
    a.m_rec = P->m_rec;
    const int64_t units = (int64_t)P->R * P->Hkv * a.n_slabs;
    // Warps per unit: split a unit's partials over more warps only while the
    // whole grid stays under about 8 warps per SM and every warp still gets
    // two partials or more on average (a sweep of 8, 16 and 32 warps per SM on
    // the four large workloads favoured 8: extra warps per unit cost more in
    // the combine than they save when units are plentiful).
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t pairs = (int64_t)P->R * P->Hq;
    const int64_t n_part = (int64_t)P->hdr.n_prefix_partials + P->hdr.n_suffix_partials;
    const double per_pair = pairs > 0 ? (double)n_part / (double)pairs : 0.0;
    int W = 1;
    while (W < kWarps && units * W < (int64_t)sms * 8 && 2.0 * W <= per_pair) W *= 2;
    a.W = W;
    const int64_t per_cta = kWarps / W;
    const int grid = (int)((units + per_cta - 1) / per_cta);
    if (grid == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(32 * kWarps);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_pass ? 1 : 0;
    return P->D == 128 ? cudaLaunchKernelEx(&cfg, k_merge<128>, a) : cudaLaunchKernelEx(&cfg, k_merge<64>, a);
}

}  // namespace fca
