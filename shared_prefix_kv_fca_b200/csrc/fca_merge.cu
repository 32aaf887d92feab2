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
// Every pass writes the G query heads of one (request, KV head, chunk) as G
// consecutive partial rows.  The kernel reads a few KB per output row block,
// each behind a lookup of where its rows lie, so it is bound by memory
// latency and by instructions, not by bandwidth; it is laid out for two
// rounds of loads per unit of work and few instructions per row:
//   - a warp takes HB query heads of one (request r, KV head h), a unit;
//     the grid is persistent (4 CTAs of 8 warps per SM), a warp taking
//     units w, w + all warps, ..., a request's units on neighbouring warps;
//   - lookup (first round): one lane per entry of the request's chain.  The
//     planner records where each group partial lies (m_rec, up to kMergeRec),
//     read together with the request's own-chunk count and first row; deeper
//     chains (and plans without records) walk the chain, and a warp scan turns
//     chunk counts into partial offsets;
//   - second round: lane k loads the HB lse values of partial k and, at the
//     same time, every lane its four columns of the first KK partials'
//     rows; the maximum and the weight sum of each head take log2(n)
//     shuffle steps over the n lanes that hold partials; further rows are
//     read KK at a time.  (HB, KK) = (2, 2) for a few partials a row, (1, 8)
//     for many (64 registers, 4 CTAs of 8 warps per SM).  Where G is a power
//     of two and rows have few partials, a warp takes a whole KV head
//     instead (merge_kv_unit: one load for every lse of the request).
// Requests with more than 32 partials, or chains longer than 32 groups, take
// a per-head loop over batches of 32 partials with a running maximum.
// Partials with lse = -inf (empty chunks) never contribute: their rows may
// hold anything, their weight is zero and they are not added.
#include <algorithm>

#include <cuda_bf16.h>

#include "fca_device.cuh"
#include "fca_internal.h"

namespace fca {

struct MergeArgs {
    int32_t R, Hq, Hkv, G, n_hb;
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

constexpr int kWarps = 8;       // warps per CTA
constexpr int kCtasPerSM = 4;     // resident CTAs per SM (the persistent grid)
constexpr int kCtasPerSMKv = 4;   // the same for whole KV heads a warp
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ int32_t warp_incl_scan(int32_t v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// Where the partial rows of (request r, KV head h) lie: entry e (held by lane
// e) covers partials [end - nch, end), the row of head 0 of its k-th being
// base + k * step.
struct Entries {
    int32_t nch, base, step, end;
    int32_t n, depth, c0, nsc, spart;
    bool wide;   // every entry fits one lane (else the rows are found serially)
};

__device__ __forceinline__ Entries lookup(const MergeArgs& a, int32_t r, int32_t h, int lane) {
    Entries E;
    E.nsc = __ldg(a.s_nch + r);
    E.spart = __ldg(a.s_part + r);
    const int32_t ng = a.m_ng ? __ldg(a.m_ng + r) : kMergeRec + 1;
    // (read whatever the count is, so that it does not wait for the count)
    const int2 rec = (a.m_rec && lane < kMergeRec) ? __ldg(a.m_rec + r * kMergeRec + lane) : make_int2(0, 0);
    const bool recorded = ng <= kMergeRec;
    E.c0 = recorded ? 0 : __ldg(a.chain_off + r);
    E.depth = recorded ? ng : __ldg(a.chain_off + r + 1) - E.c0;
    E.wide = E.depth < 32;   // warp-uniform
    E.nch = 0;
    E.base = 0;
    E.step = 0;
    if (recorded) {
        if (lane < E.depth) {
            E.nch = 1;
            E.base = rec.x + h * rec.y;
        }
    } else if (E.wide && lane < E.depth) {
        // group chain[e]: row of chunk k = g_part + ((h nch + k) nm + pos) G
        const int32_t g = __ldg(a.chain_g + E.c0 + lane), pos = __ldg(a.chain_pos + E.c0 + lane);
        const int32_t nch = __ldg(a.g_nch + g), nm = __ldg(a.g_nm + g);
        E.nch = nch;
        E.base = __ldg(a.g_part + g) + ((h * nch) * nm + pos) * a.G;
        E.step = nm * a.G;
    }
    if (E.wide && lane == E.depth) {   // own chunks: row of chunk k = s_part + (h nsc + k) G
        E.nch = E.nsc;
        E.base = E.spart + h * E.nsc * a.G;
        E.step = a.G;
    }
    E.end = warp_incl_scan(E.nch, lane);
    if (E.wide) {
        E.n = __shfl_sync(kFull, E.end, E.depth);
    } else {   // (never for a recorded request: depth <= kMergeRec)
        E.n = E.nsc;
        for (int32_t c = E.c0; c < E.c0 + E.depth; ++c) E.n += __ldg(a.g_nch + __ldg(a.chain_g + c));
    }
    return E;
}

// Row of head 0 of partial k (any k < n; every lane calls, with its own k).
__device__ __forceinline__ int32_t partial_row(const MergeArgs& a, const Entries& E, int32_t h, int32_t k) {
    if (E.wide) {
        int32_t e = 0;
        for (int32_t x = 0; x < E.depth; ++x) e += (k >= __shfl_sync(kFull, E.end, x)) ? 1 : 0;
        const int32_t end = __shfl_sync(kFull, E.end, e);
        const int32_t cnt = __shfl_sync(kFull, E.nch, e);
        const int32_t base = __shfl_sync(kFull, E.base, e);
        const int32_t step = __shfl_sync(kFull, E.step, e);
        return base + (k - (end - cnt)) * step;
    }
    if (k >= E.n) return 0;
    for (int32_t c = E.c0; c < E.c0 + E.depth; ++c) {
        const int32_t g = __ldg(a.chain_g + c), nch = __ldg(a.g_nch + g);
        if (k < nch) return __ldg(a.g_part + g) + ((h * nch + k) * __ldg(a.g_nm + g) + __ldg(a.chain_pos + c)) * a.G;
        k -= nch;
    }
    return E.spart + (h * E.nsc + k) * a.G;
}

template <int D>
__device__ __forceinline__ void store_row(const MergeArgs& a, int32_t q, float4 acc, float m, float l, int lane) {
    const float inv = l > 0.f ? __frcp_rn(l) : 0.f;
    if (lane < D / 4) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
        uint2 v;
        v.x = *reinterpret_cast<uint32_t*>(&lo);
        v.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(a.out + (int64_t)q * D + lane * 4) = v;
    }
    if (a.lse && lane == 0) a.lse[q] = l > 0.f ? m + __logf(l) : -INFINITY;
}

__device__ __forceinline__ void fma4(float4& acc, float w, const float4& v) {
    acc.x = fmaf(w, v.x, acc.x);
    acc.y = fmaf(w, v.y, acc.y);
    acc.z = fmaf(w, v.z, acc.z);
    acc.w = fmaf(w, v.w, acc.w);
}

}  // namespace

// Query heads gq0 .. gq0 + HB - 1 of (request r, KV head h): one warp.
template <int D, int HB, int KK>
__device__ __forceinline__ void merge_unit(const MergeArgs& a, int32_t r, int32_t h, int32_t gq0, int lane) {
    const int32_t nh = min(HB, a.G - gq0);   // heads of this block
    const int32_t q0 = r * a.Hq + h * a.G + gq0;   // its first output row
    const bool cols = lane < D / 4;
    const Entries E = lookup(a, r, h, lane);
    const int32_t n = E.n;

    if (E.wide && n <= 32) {
        // ---- lane k < n holds partial k
        const int32_t row = partial_row(a, E, h, lane) + gq0;
        float lk[HB];
#pragma unroll
        for (int j = 0; j < HB; ++j) lk[j] = (lane < n && j < nh) ? __ldg(a.part_lse + row + j) : -INFINITY;
        float4 o[KK][HB];
        auto load_rows = [&](int32_t k0) {
#pragma unroll
            for (int u = 0; u < KK; ++u) {
                const int32_t ru = __shfl_sync(kFull, row, (k0 + u) & 31);
                const float* src = a.part_o + (int64_t)ru * D + lane * 4;
#pragma unroll
                for (int j = 0; j < HB; ++j)
                    o[u][j] = (k0 + u < n && j < nh && cols) ? __ldg(reinterpret_cast<const float4*>(src + j * D))
                                                              : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        };
        load_rows(0);
        // each head's maximum and weight sum over lanes [0, n): xor steps
        // within the smallest power of two holding n, then from lane 0
        float m[HB], l[HB], w[HB];
#pragma unroll
        for (int j = 0; j < HB; ++j) {
            float mx = lk[j];
            for (int s = 1; s < n; s <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, s));
            w[j] = lk[j] == -INFINITY ? 0.f : __expf(lk[j] - mx);
            float sm = w[j];
            for (int s = 1; s < n; s <<= 1) sm += __shfl_xor_sync(kFull, sm, s);
            m[j] = __shfl_sync(kFull, mx, 0);
            l[j] = __shfl_sync(kFull, sm, 0);
        }
        float4 acc[HB];
#pragma unroll
        for (int j = 0; j < HB; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int32_t k0 = 0; k0 < n; k0 += KK) {
            if (k0 > 0) load_rows(k0);
#pragma unroll
            for (int u = 0; u < KK; ++u)
#pragma unroll
                for (int j = 0; j < HB; ++j) {
                    const float wu = __shfl_sync(kFull, w[j], (k0 + u) & 31);
                    if (k0 + u < n && wu > 0.f) fma4(acc[j], wu, o[u][j]);
                }
        }
#pragma unroll
        for (int j = 0; j < HB; ++j)
            if (j < nh) store_row<D>(a, q0 + j, acc[j], m[j], l[j], lane);
        return;
    }

    // ---- many partials or a deep chain: one head at a time, batches of 32
    for (int j = 0; j < nh; ++j) {
        float m = -INFINITY, l = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int32_t b0 = 0; b0 < n; b0 += 32) {
            const int32_t k = b0 + lane;
            const int32_t row = partial_row(a, E, h, k) + gq0 + j;
            const float lk = k < n ? __ldg(a.part_lse + row) : -INFINITY;
            float mb = lk;
#pragma unroll
            for (int s = 16; s > 0; s >>= 1) mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, s));
            const float m_new = fmaxf(m, mb);
            const float sc = m_new == -INFINITY ? 1.f : __expf(m - m_new);   // 0 while nothing has been added
            const float w = lk == -INFINITY ? 0.f : __expf(lk - m_new);
            float ws = w;
#pragma unroll
            for (int s = 16; s > 0; s >>= 1) ws += __shfl_xor_sync(kFull, ws, s);
            l = l * sc + ws;
            m = m_new;
            acc.x *= sc; acc.y *= sc; acc.z *= sc; acc.w *= sc;
            const int32_t nb = min(32, n - b0);
            for (int32_t u = 0; u < nb; ++u) {
                const int32_t ru = __shfl_sync(kFull, row, u);
                const float wu = __shfl_sync(kFull, w, u);
                if (wu > 0.f && cols)
                    fma4(acc, wu, __ldg(reinterpret_cast<const float4*>(a.part_o + (int64_t)ru * D + lane * 4)));
            }
        }
        store_row<D>(a, q0 + j, acc, m, l, lane);
    }
}

// All G query heads of (request r, KV head h), G a power of two, when the
// request has at most 32 / G partials: lane k G + i holds head i of partial
// k, so one load gives every lse, and each head's maximum and weight sum take
// log2(n) shuffle steps over lanes G apart; the rows are then read four heads
// of one partial at a time (64 registers: 4 CTAs per SM).  Otherwise the unit
// goes to merge_unit, two heads at a time.
template <int D>
__device__ __forceinline__ void merge_kv_unit(const MergeArgs& a, int32_t r, int32_t h, int lane) {
    constexpr int KK = 1;
    const int32_t G = a.G;
    const Entries E = lookup(a, r, h, lane);
    const int32_t n = E.n;
    if (!E.wide || n * G > 32) {
        for (int32_t gq0 = 0; gq0 < G; gq0 += 2) merge_unit<D, 2, 2>(a, r, h, gq0, lane);
        return;
    }
    const int32_t lg = __ffs(G) - 1;   // log2 G
    const int32_t kl = lane >> lg, il = lane & (G - 1);
    const int32_t row = partial_row(a, E, h, kl);   // head 0's row of partial kl (lanes kl < n)
    const float lk = lane < n * G ? __ldg(a.part_lse + row + il) : -INFINITY;
    const bool cols = lane < D / 4;
    float4 o[KK][4];
    auto load_rows = [&](int32_t b0, int32_t k0) {
#pragma unroll
        for (int u = 0; u < KK; ++u) {
            const int32_t ru = __shfl_sync(kFull, row, ((k0 + u) << lg) & 31);
            const float* src = a.part_o + ((int64_t)ru + b0) * D + lane * 4;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                o[u][j] = (k0 + u < n && b0 + j < G && cols) ? __ldg(reinterpret_cast<const float4*>(src + j * D))
                                                              : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    load_rows(0, 0);
    float mx = lk;
    for (int s = G; s < G * n; s <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, s));
    const float w = lk == -INFINITY ? 0.f : __expf(lk - mx);
    float sm = w;
    for (int s = G; s < G * n; s <<= 1) sm += __shfl_xor_sync(kFull, sm, s);
    // lanes i < G (partial 0) hold head i's maximum and sum
    const int32_t q0 = r * a.Hq + h * G;
    for (int32_t b0 = 0; b0 < G; b0 += 4) {
        float4 acc[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int32_t k0 = 0; k0 < n; k0 += KK) {
            if (b0 > 0 || k0 > 0) load_rows(b0, k0);
#pragma unroll
            for (int u = 0; u < KK; ++u)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float wu = __shfl_sync(kFull, w, (((k0 + u) << lg) + b0 + j) & 31);
                    if (k0 + u < n && b0 + j < G && wu > 0.f) fma4(acc[j], wu, o[u][j]);
                }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float mj = __shfl_sync(kFull, mx, (b0 + j) & 31), lj = __shfl_sync(kFull, sm, (b0 + j) & 31);
            if (b0 + j < G) store_row<D>(a, q0 + b0 + j, acc[j], mj, lj, lane);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(32 * kWarps, kCtasPerSMKv) k_merge_kv(MergeArgs a) {
    dev::pdl_wait();   // (as k_merge)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t n_units = a.R * a.Hkv;
    for (int32_t u = blockIdx.x * kWarps + warp; u < n_units; u += gridDim.x * kWarps) {
        const int32_t r = u / a.Hkv;
        merge_kv_unit<D>(a, r, u - r * a.Hkv, lane);
    }
}

template <int D, int HB, int KK>
__global__ void __launch_bounds__(32 * kWarps, kCtasPerSM) k_merge(MergeArgs a) {
    // launched after a pass with programmatic serialization: its rows are
    // complete and visible past this point
    dev::pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // persistent: warp w takes units w, w + all warps, ...; unit u is head
    // block y = u mod Y of request u / Y, Y = Hkv x head blocks (a request's
    // units on neighbouring warps)
    const int32_t Y = a.Hkv * a.n_hb, n_units = a.R * Y;
    for (int32_t u = blockIdx.x * kWarps + warp; u < n_units; u += gridDim.x * kWarps) {
        const int32_t r = u / Y, y = u - r * Y;
        const int32_t h = y / a.n_hb;
        merge_unit<D, HB, KK>(a, r, h, (y - h * a.n_hb) * HB, lane);
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
    if (P->R == 0) return cudaSuccess;
    // partials per output row on average: many -> one head a warp, eight rows in flight
    const int64_t pairs = (int64_t)P->R * P->Hq;
    const int64_t n_part = (int64_t)P->hdr.n_prefix_partials + P->hdr.n_suffix_partials;
    const bool many = pairs > 0 && n_part > 4 * pairs;
    // whole KV heads a warp where G is a power of two (few partials a row)
    const bool kv = !many && P->G <= 16 && (P->G & (P->G - 1)) == 0;
    const int hb = many ? 1 : kv ? P->G : 2;
    a.n_hb = (P->G + hb - 1) / hb;
    cudaLaunchConfig_t cfg = {};
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t units = (int64_t)P->R * P->Hkv * a.n_hb;
    cfg.gridDim = dim3((unsigned)std::min<int64_t>((units + kWarps - 1) / kWarps,
                                                   (int64_t)sms * (kv ? kCtasPerSMKv : kCtasPerSM)));
    cfg.blockDim = dim3(32 * kWarps);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_pass ? 1 : 0;
    if (P->D == 128)
        return many ? cudaLaunchKernelEx(&cfg, k_merge<128, 1, 8>, a)
               : kv ? cudaLaunchKernelEx(&cfg, k_merge_kv<128>, a)
                    : cudaLaunchKernelEx(&cfg, k_merge<128, 2, 2>, a);
    return many ? cudaLaunchKernelEx(&cfg, k_merge<64, 1, 8>, a)
           : kv ? cudaLaunchKernelEx(&cfg, k_merge_kv<64>, a)
                : cudaLaunchKernelEx(&cfg, k_merge<64, 2, 2>, a);
}

}  // namespace fca
