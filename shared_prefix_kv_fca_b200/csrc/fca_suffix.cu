// Per-request pass over a request's own KV blocks (split-KV decode).
//
// "ZoRRo Inference & Forest Cascade Attention", "Core Mechanism" step 2,
// second bullet: one pass per request over its unique suffix blocks.  The
// same kernel over a request's whole table is the flat paged decode that FCA
// is measured against (standard attention, which reads every shared block
// once per request, "Overview").
//
// One CTA per work item = (request, KV head, token chunk).  Warp 0 streams
// the chunk's paged blocks into a ring of shared-memory slots with TMA
// (one 16-token x head_dim tile of K and one of V per slot, 128-byte
// swizzle so that the consumers' strided reads are bank-conflict free).
// Warps 1-4 take slots round-robin; each keeps its own online-softmax state
// for the G query heads of the KV head:
//   - QK: lane = (token t, half of the query rows); full-length dot products
//     against the pre-scaled fp32 queries in shared memory; softmax maxima and
//     sums by warp shuffles over the 16 token lanes;
//   - PV: lane = head_dim slice; probabilities broadcast from shared memory.
// The four warp states are merged once at the end and written as G partial
// rows (normalised o, natural-log lse) for the merge pass.
#include <cuda_bf16.h>

#include "fca_device.cuh"
#include "fca_internal.h"

namespace fca {

namespace {

constexpr int kSufSlots = 8;
constexpr int kSufThreads = 160;

struct SuffixArgs {
    const SuffixItem* items;
    const int32_t* bt;
    int32_t max_blocks, num_blocks, Hq, G;
    const __nv_bfloat16* q;
    float q_scale;            // scale * log2(e)
    float* part_o;
    float* part_lse;
    int32_t* err;
};

template <int D, int GM>
struct SufLayout {
    static constexpr int kHalves = D / 64;
    static constexpr int kTile = kHalves * 16 * 128;          // one 16-token K (or V) tile
    static constexpr int kSlot = 2 * kTile;
    static constexpr int kRing = kSufSlots * kSlot;
    static constexpr int kQ = GM * D * 4;                     // fp32 queries
    static constexpr int kP = 4 * (16 * GM + GM) * 4;         // per-warp p[16][GM] + alpha[GM]
    static constexpr int kComb = 4 * GM * (D + 2) * 4;        // per-warp o, m, l
    static constexpr int kBars = 2 * kSufSlots * 8 + 16;
    static constexpr int kTotal = kRing + kQ + kP + kComb + kBars + 1024;   // + alignment slack
};

template <int D, int GM>
__global__ void __launch_bounds__(kSufThreads) k_suffix(SuffixArgs a, const __grid_constant__ CUtensorMap tmK,
                                                        const __grid_constant__ CUtensorMap tmV) {
    using L = SufLayout<D, GM>;
    constexpr int RPL = GM / 2;     // query rows per lane (two row halves)
    constexpr int DPL = D / 32;     // head_dim elements per lane in PV
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    float* qs = reinterpret_cast<float*>(smem + L::kRing);
    float* ps = reinterpret_cast<float*>(smem + L::kRing + L::kQ);
    float* comb = reinterpret_cast<float*>(smem + L::kRing + L::kQ + L::kP);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kRing + L::kQ + L::kP + L::kComb);
    uint64_t* empty = full + kSufSlots;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kSufSlots);

    const SuffixItem it = a.items[blockIdx.x];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t blk0 = it.tok0 / kBlockSize;
    const int32_t nblk = (it.tok1 + kBlockSize - 1) / kBlockSize - blk0;
    const int32_t* row = a.bt + (int64_t)it.request * a.max_blocks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSufSlots; ++s) {
            dev::mbar_init(&full[s], 1);
            dev::mbar_init(&empty[s], 1);
        }
        *abort_flag = 0;
        dev::fence_mbarrier_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------- producer
        if (lane == 0) {
            dev::tma_prefetch_desc(&tmK);
            dev::tma_prefetch_desc(&tmV);
            int32_t issued = 0;
            for (int32_t j = 0; j < nblk; ++j) {
                const int s = j % kSufSlots;
                if (j >= kSufSlots &&
                    !dev::mbar_wait(&empty[s], ((j / kSufSlots) - 1) & 1, abort_flag, a.err))
                    break;
                const int32_t phys = row[blk0 + j];
                uint8_t* kdst = ring + s * L::kSlot;
                uint8_t* vdst = kdst + L::kTile;
                dev::mbar_arrive_expect_tx(&full[s], 2 * L::kTile);
#pragma unroll
                for (int hf = 0; hf < L::kHalves; ++hf) {
                    dev::tma_load_3d(kdst + hf * 2048, &tmK, &full[s], hf * 64, it.head, phys * kBlockSize);
                    dev::tma_load_3d(vdst + hf * 2048, &tmV, &full[s], hf * 64, it.head, phys * kBlockSize);
                }
                ++issued;
            }
            // never leave with copies in flight
            for (int32_t j = issued - 1; j >= 0 && j >= issued - kSufSlots; --j) {
                volatile int never = 0;
                dev::mbar_wait(&full[j % kSufSlots], (j / kSufSlots) & 1, &never, a.err);
            }
        }
        __syncwarp();
    } else {
        // ---------------- consumers
        const int cw = warp - 1;
        const int ctid = threadIdx.x - 32;
        // queries, pre-scaled into the log2 domain; padded rows are zero
        for (int i = ctid; i < GM * D; i += 128) {
            const int g = i / D, d = i % D;
            float v = 0.f;
            if (g < a.G)
                v = __bfloat162float(a.q[((int64_t)it.request * a.Hq + it.head * a.G + g) * D + d]) * a.q_scale;
            qs[i] = v;
        }
        dev::named_barrier_sync(1, 128);

        const int t = lane & 15, hr = lane >> 4;
        float m_run[RPL], l_run[RPL];
#pragma unroll
        for (int j = 0; j < RPL; ++j) {
            m_run[j] = -INFINITY;
            l_run[j] = 0.f;
        }
        float o[GM][DPL];
#pragma unroll
        for (int g = 0; g < GM; ++g)
#pragma unroll
            for (int e = 0; e < DPL; ++e) o[g][e] = 0.f;
        float* pw = ps + cw * (16 * GM + GM);     // this warp's p[16][GM], alpha[GM]
        float* aw = pw + 16 * GM;

        for (int32_t j = cw; j < nblk; j += 4) {
            const int s = j % kSufSlots;
            if (!dev::mbar_wait(&full[s], (j / kSufSlots) & 1, abort_flag, a.err)) break;
            const uint8_t* kt = ring + s * L::kSlot;
            const uint8_t* vt = kt + L::kTile;
            const int32_t tok = (blk0 + j) * kBlockSize + t;
            const int32_t nvalid = min(kBlockSize, it.tok1 - (blk0 + j) * kBlockSize);

            // scores for (token t, rows hr*RPL + jj)
            float sc[RPL];
#pragma unroll
            for (int jj = 0; jj < RPL; ++jj) sc[jj] = 0.f;
#pragma unroll 4
            for (int c = 0; c < D / 8; ++c) {
                const int hf = c >> 3, cc = c & 7;
                const uint4 kv = *reinterpret_cast<const uint4*>(kt + hf * 2048 + t * 128 + ((cc ^ (t & 7)) << 4));
                float kf[8];
                kf[0] = dev::bf16_lo(kv.x); kf[1] = dev::bf16_hi(kv.x);
                kf[2] = dev::bf16_lo(kv.y); kf[3] = dev::bf16_hi(kv.y);
                kf[4] = dev::bf16_lo(kv.z); kf[5] = dev::bf16_hi(kv.z);
                kf[6] = dev::bf16_lo(kv.w); kf[7] = dev::bf16_hi(kv.w);
#pragma unroll
                for (int jj = 0; jj < RPL; ++jj) {
                    const float* qr = qs + (hr * RPL + jj) * D + c * 8;
                    const float4 q0 = *reinterpret_cast<const float4*>(qr);
                    const float4 q1 = *reinterpret_cast<const float4*>(qr + 4);
                    float acc = sc[jj];
                    acc = fmaf(q0.x, kf[0], acc); acc = fmaf(q0.y, kf[1], acc);
                    acc = fmaf(q0.z, kf[2], acc); acc = fmaf(q0.w, kf[3], acc);
                    acc = fmaf(q1.x, kf[4], acc); acc = fmaf(q1.y, kf[5], acc);
                    acc = fmaf(q1.z, kf[6], acc); acc = fmaf(q1.w, kf[7], acc);
                    sc[jj] = acc;
                }
            }
            const bool valid = tok < it.tok1;
#pragma unroll
            for (int jj = 0; jj < RPL; ++jj) {
                float x = valid ? sc[jj] : -INFINITY;
                float mx = x;
#pragma unroll
                for (int off = 1; off < 16; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                const float m_new = fmaxf(m_run[jj], mx);
                const float alpha = exp2f(m_run[jj] - m_new);
                const float p = valid ? exp2f(x - m_new) : 0.f;
                float ps_sum = p;
#pragma unroll
                for (int off = 1; off < 16; off <<= 1) ps_sum += __shfl_xor_sync(0xffffffffu, ps_sum, off);
                l_run[jj] = l_run[jj] * alpha + ps_sum;
                m_run[jj] = m_new;
                pw[t * GM + hr * RPL + jj] = p;
                if (t == 0) aw[hr * RPL + jj] = alpha;
            }
            __syncwarp();
            // o = o * alpha + sum_t p_t v_t over this lane's head_dim slice
#pragma unroll
            for (int g = 0; g < GM; ++g) {
                const float al = aw[g];
#pragma unroll
                for (int e = 0; e < DPL; ++e) o[g][e] *= al;
            }
            const int e0 = lane * DPL;                // first element of the slice
            const int hf = e0 >> 6, byte_in_half = (e0 & 63) * 2;
            for (int tt = 0; tt < nvalid; ++tt) {
                const uint8_t* vrow = vt + hf * 2048 + tt * 128;
                const int chunk = byte_in_half >> 4, within = byte_in_half & 15;
                const uint8_t* vp = vrow + ((chunk ^ (tt & 7)) << 4) + within;
                float vf[DPL];
                if constexpr (DPL == 4) {
                    const uint2 vv = *reinterpret_cast<const uint2*>(vp);
                    vf[0] = dev::bf16_lo(vv.x); vf[1] = dev::bf16_hi(vv.x);
                    vf[2] = dev::bf16_lo(vv.y); vf[3] = dev::bf16_hi(vv.y);
                } else {
                    const uint32_t vv = *reinterpret_cast<const uint32_t*>(vp);
                    vf[0] = dev::bf16_lo(vv); vf[1] = dev::bf16_hi(vv);
                }
                const float* prow = pw + tt * GM;
#pragma unroll
                for (int g = 0; g < GM; ++g) {
                    const float p = prow[g];
#pragma unroll
                    for (int e = 0; e < DPL; ++e) o[g][e] = fmaf(p, vf[e], o[g][e]);
                }
            }
            __syncwarp();
            if (lane == 0) dev::mbar_arrive(&empty[s]);
        }

        // ---------------- merge the four warp states, write G partial rows
        float* cm = comb;                       // [4][GM] m
        float* cl = comb + 4 * GM;              // [4][GM] l
        float* co = comb + 8 * GM;              // [4][GM][D] o
        if (t == 0) {
#pragma unroll
            for (int jj = 0; jj < RPL; ++jj) {
                cm[cw * GM + hr * RPL + jj] = m_run[jj];
                cl[cw * GM + hr * RPL + jj] = l_run[jj];
            }
        }
#pragma unroll
        for (int g = 0; g < GM; ++g)
#pragma unroll
            for (int e = 0; e < DPL; ++e) co[(cw * GM + g) * D + lane * DPL + e] = o[g][e];
        dev::named_barrier_sync(1, 128);
        for (int i = ctid; i < a.G * D; i += 128) {
            const int g = i / D, d = i % D;
            float m = -INFINITY;
#pragma unroll
            for (int w = 0; w < 4; ++w) m = fmaxf(m, cm[w * GM + g]);
            float l = 0.f, acc = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float mw = cm[w * GM + g];
                if (mw == -INFINITY) continue;
                const float sc = exp2f(mw - m);
                l += cl[w * GM + g] * sc;
                acc += co[(w * GM + g) * D + d] * sc;
            }
            const int64_t prow = it.part_row0 + g;
            a.part_o[prow * D + d] = acc / l;
            if (d == 0) a.part_lse[prow] = (m + log2f(l)) * 0.69314718055994531f;
        }
    }
}

template <int D, int GM>
cudaError_t launch_suffix_t(const fca_plan_s* P, const SuffixArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                            int n_items, cudaStream_t stream) {
    using L = SufLayout<D, GM>;
    cudaError_t e = cudaFuncSetAttribute(k_suffix<D, GM>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal);
    if (e != cudaSuccess) return e;
    k_suffix<D, GM><<<n_items, kSufThreads, L::kTotal, stream>>>(a, tk, tv);
    (void)P;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_suffix(const fca_plan_s* P, const void* q, const CUtensorMap& tk, const CUtensorMap& tv,
                          float scale, cudaStream_t stream) {
    const int n = P->hdr.n_suffix_items;
    if (n == 0) return cudaSuccess;
    SuffixArgs a;
    a.items = P->suffix_items;
    a.bt = P->bt;
    a.max_blocks = P->max_blocks;
    a.num_blocks = P->num_blocks;
    a.Hq = P->Hq;
    a.G = P->G;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.q_scale = scale * 1.4426950408889634f;
    a.part_o = P->part_o;
    a.part_lse = P->part_lse;
    a.err = P->dev_status;
    const int G = P->G;
    if (P->D == 128) {
        if (G <= 2) return launch_suffix_t<128, 2>(P, a, tk, tv, n, stream);
        if (G <= 4) return launch_suffix_t<128, 4>(P, a, tk, tv, n, stream);
        if (G <= 8) return launch_suffix_t<128, 8>(P, a, tk, tv, n, stream);
        return launch_suffix_t<128, 16>(P, a, tk, tv, n, stream);
    }
    if (G <= 2) return launch_suffix_t<64, 2>(P, a, tk, tv, n, stream);
    if (G <= 4) return launch_suffix_t<64, 4>(P, a, tk, tv, n, stream);
    if (G <= 8) return launch_suffix_t<64, 8>(P, a, tk, tv, n, stream);
    return launch_suffix_t<64, 16>(P, a, tk, tv, n, stream);
}

}  // namespace fca
