// Per-request pass over a request's own KV blocks (split-KV decode).
//
// "ZoRRo Inference & Forest Cascade Attention", "Core Mechanism" step 2,
// second bullet: one pass per request over its unique suffix blocks.  The
// same kernel over a request's whole table is the flat paged decode that FCA
// is measured against (standard attention, which reads every shared block
// once per request, "Overview").
//
// Work item = (request, KV head, token chunk); one warp owns one item at a
// time and keeps everything to itself, so warps never wait for each other:
//   - its lane 0 streams the chunk's paged 16-token blocks (K and V tiles of
//     one head, 128-byte swizzle) into the warp's own ring of kSlots
//     shared-memory slots with TMA, refilling a slot as soon as the warp has
//     consumed it;
//   - the G query heads that share the KV head are the N side of warp MMAs
//     (mma.sync m16n8k16, bf16 in, fp32 accumulate) with the block's 16
//     tokens on the M side: S^T = K Q^T, then O^T += V^T P^T.  Each lane
//     holds two query columns, so the online softmax (column max over the
//     block by three shuffles, per-lane running sums) and the O rescale stay
//     in registers; P^T reaches the second MMA through movmatrix;
//   - at the end of the chunk it writes G partial rows (normalised o,
//     natural-log lse) for the merge pass.
// Items are taken longest first from a global counter; the last warp out
// resets the counter for the next launch.
#include <algorithm>

#include <cuda_bf16.h>

#include "fca_device.cuh"
#include "fca_internal.h"

namespace fca {

namespace {

constexpr int kSufWarps = 8;

struct SuffixArgs {
    const SuffixItem* items;
    int32_t n_items;
    const int32_t* bt;
    int32_t max_blocks, Hq, G;
    const __nv_bfloat16* q;
    float scale_log2;
    float* part_o;
    float* part_lse;
    int32_t* err;
    int32_t* sched;           // [0] next item, [1] warps done
};

template <int D>
struct SufLayout {
    static constexpr int kSlots = D == 128 ? 3 : 6;
    static constexpr int kTile = (D / 64) * 16 * 128;     // one 16-token tile of K (or V), bytes
    static constexpr int kSlot = 2 * kTile;
    static constexpr int kWarpRing = kSlots * kSlot;
    static constexpr int kBars = kSufWarps * kSlots * 8;
    static constexpr int kTotal = kSufWarps * kWarpRing + kBars + 1024;
};

// Address of the 16-byte chunk holding (token, element e..e+7) of a tile laid
// out by TMA with 128-byte swizzle: 64-element halves of 16 rows x 128 B.
__device__ __forceinline__ uint32_t tile_chunk(uint32_t tile, int tok, int e) {
    return tile + (e >> 6) * 2048 + tok * 128 + ((((e & 63) >> 3) ^ (tok & 7)) << 4);
}

// kDevCount: the item count is read from sched[2], written on the device by
// the kernel that built the items (a.n_items is then only the bound the grid
// was sized for).
template <int D, int NT, bool kDevCount>
__global__ void __launch_bounds__(kSufWarps * 32, 1)
    k_suffix(SuffixArgs a, const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
    using L = SufLayout<D>;
    constexpr int KS = D / 16;        // k-steps of Q K^T, m-tiles of V^T P^T
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, tig = lane & 3;
    uint8_t* ring = smem + warp * L::kWarpRing;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSufWarps * L::kWarpRing) + warp * L::kSlots;
    const uint32_t ring_u32 = dev::smem_u32(ring);

    if (lane == 0) {
        for (int s = 0; s < L::kSlots; ++s) dev::mbar_init(&full[s], 1);
        dev::fence_mbarrier_init();
        dev::tma_prefetch_desc(&tmK);
        dev::tma_prefetch_desc(&tmV);
    }
    __syncwarp();
    volatile int no_abort = 0;
    const int32_t n_items = kDevCount ? *reinterpret_cast<volatile const int32_t*>(a.sched + 2) : a.n_items;
    uint32_t uses = 0;        // blocks this warp has pushed through its ring so far
    bool failed = false;

    while (!failed) {
        int32_t idx = 0;
        if (lane == 0) idx = atomicAdd(&a.sched[0], 1);
        idx = __shfl_sync(0xffffffffu, idx, 0);
        if (idx >= n_items) {
            // every item is taken: the merge may be set up (it waits for this
            // grid to end before it reads a row)
            dev::pdl_launch_dependents();
            break;
        }
        const SuffixItem it = a.items[idx];
        const int32_t blk0 = it.tok0 / kBlockSize;
        const int32_t nblk = (it.tok1 + kBlockSize - 1) / kBlockSize - blk0;
        const int32_t* row = a.bt + (int64_t)it.request * a.max_blocks + blk0;

        // Block ids in registers, 32 at a time: lane l holds block 32 b + l of
        // batch b (the current batch and the next; the next is read when the
        // current one starts, long before it is needed), so no table lookup
        // sits on lane 0's issue path.
        auto bid_load = [&](int32_t b) -> int32_t {
            const int32_t jj = b * 32 + lane;
            return jj < nblk ? __ldg(row + jj) : 0;
        };
        int32_t bid_cur = bid_load(0), bid_nxt = nblk > 32 ? bid_load(1) : 0;
        // id of block jj, which lies in batch `base` or the one after (all lanes call)
        auto bid_of = [&](int32_t jj, int32_t base) -> int32_t {
            const int32_t vc = __shfl_sync(0xffffffffu, bid_cur, jj & 31);
            const int32_t vn = __shfl_sync(0xffffffffu, bid_nxt, jj & 31);
            return (jj >> 5) == base ? vc : vn;
        };
        auto issue = [&](int32_t j, int32_t bid) {   // lane 0: block j of the item into its slot
            const uint32_t u = uses + j;
            const int s = u % L::kSlots;
            const int32_t trow = bid * kBlockSize;
            uint8_t* kdst = ring + s * L::kSlot;
            dev::fence_proxy_async_smem();
            dev::mbar_arrive_expect_tx(&full[s], L::kSlot);
#pragma unroll
            for (int hf = 0; hf < D / 64; ++hf) {
                dev::tma_load_3d(kdst + hf * 2048, &tmK, &full[s], hf * 64, it.head, trow);
                dev::tma_load_3d(kdst + L::kTile + hf * 2048, &tmV, &full[s], hf * 64, it.head, trow);
            }
        };
#pragma unroll
        for (int32_t j = 0; j < L::kSlots; ++j) {
            const int32_t bid = bid_of(j, 0);
            if (lane == 0 && j < nblk) issue(j, bid);
        }

        // Q^T fragments (B operand): column n = query head nt * 8 + g8,
        // rows k = head_dim pairs 16 ks + 2 tig (+8).  Heads past G are zero.
        uint32_t qb[NT][KS][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int qh = nt * 8 + g8;
            const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
                a.q + ((int64_t)it.request * a.Hq + it.head * a.G + (qh < a.G ? qh : 0)) * D);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                qb[nt][ks][0] = qh < a.G ? __ldg(qrow + ks * 8 + tig) : 0u;
                qb[nt][ks][1] = qh < a.G ? __ldg(qrow + ks * 8 + 4 + tig) : 0u;
            }
        }

        float m_run[NT][2], l_run[NT][2];
        float o[NT][KS][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m_run[nt][0] = m_run[nt][1] = -INFINITY;
            l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
        }

        for (int32_t j = 0; j < nblk; ++j) {
            const uint32_t u = uses + j;
            const int s = u % L::kSlots;
            const bool got = dev::mbar_wait(&full[s], (u / L::kSlots) & 1, &no_abort, a.err);
            if (!__all_sync(0xffffffffu, got)) { failed = true; break; }
            const uint32_t kt = ring_u32 + s * L::kSlot, vt = kt + L::kTile;
            const int32_t nvalid = min(kBlockSize, it.tok1 - (blk0 + j) * kBlockSize);
            if (nvalid < kBlockSize) {
                // rows past the sequence may hold anything: P is zero there, but
                // 0 * NaN is not, so clear those V rows before the second MMA
                uint8_t* vrow = ring + s * L::kSlot + L::kTile;
                for (int c = lane; c < (kBlockSize - nvalid) * (D / 8); c += 32) {
                    const int tok = nvalid + c / (D / 8), e = (c % (D / 8)) * 8;
                    *reinterpret_cast<uint4*>(vrow + (e >> 6) * 2048 + tok * 128 + (e & 63) * 2) =
                        make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
            }

            // S^T = K Q^T: lane holds tokens g8, g8 + 8 x query columns 2 tig, 2 tig + 1
            float sc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                const int mi = lane >> 3, rr = lane & 7;
                uint32_t a0, a1, a2, a3;
                dev::ldsm_x4(tile_chunk(kt, rr + 8 * (mi & 1), ks * 16 + 8 * (mi >> 1)), a0, a1, a2, a3);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) dev::mma_bf16_16816(sc[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
            }

            uint32_t pb[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float x[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int tok = g8 + (i >> 1) * 8;
                    x[i] = tok < nvalid ? sc[nt][i] * a.scale_log2 : -INFINITY;
                }
                float alpha[2], p[4];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float mx = fmaxf(x[c], x[c + 2]);
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    const float m_new = fmaxf(m_run[nt][c], mx);
                    alpha[c] = exp2f(m_run[nt][c] - m_new);
                    m_run[nt][c] = m_new;
                    p[c] = exp2f(x[c] - m_new);
                    p[c + 2] = exp2f(x[c + 2] - m_new);
                    l_run[nt][c] = l_run[nt][c] * alpha[c] + p[c] + p[c + 2];
                }
#pragma unroll
                for (int mt = 0; mt < KS; ++mt) {
                    o[nt][mt][0] *= alpha[0];
                    o[nt][mt][1] *= alpha[1];
                    o[nt][mt][2] *= alpha[0];
                    o[nt][mt][3] *= alpha[1];
                }
                // P^T as the B operand: transpose the two 8x8 token blocks
                pb[nt][0] = dev::movmatrix_trans(dev::pack_bf16x2(p[0], p[1]));
                pb[nt][1] = dev::movmatrix_trans(dev::pack_bf16x2(p[2], p[3]));
            }

            // O^T += V^T P^T: m-tile mt covers head_dim rows 16 mt .. 16 mt + 15
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                const int mi = lane >> 3, rr = lane & 7;
                uint32_t a0, a1, a2, a3;
                dev::ldsm_x4_trans(tile_chunk(vt, rr + 8 * (mi >> 1), mt * 16 + 8 * (mi & 1)), a0, a1, a2, a3);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) dev::mma_bf16_16816(o[nt][mt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            }
            __syncwarp();
            if (((j + 1) & 31) == 0) {   // the next block starts a new batch of ids
                bid_cur = bid_nxt;
                bid_nxt = bid_load(((j + 1) >> 5) + 1);
            }
            const int32_t t = j + L::kSlots;   // the block that takes the slot just freed
            const int32_t bid_t = bid_of(t, (j + 1) >> 5);
            if (lane == 0 && t < nblk) issue(t, bid_t);
        }
        uses += nblk;
        if (failed) break;

        // column sums over the 8 lanes that share a column, then the partial rows
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float l = l_run[nt][c];
                l += __shfl_xor_sync(0xffffffffu, l, 4);
                l += __shfl_xor_sync(0xffffffffu, l, 8);
                l += __shfl_xor_sync(0xffffffffu, l, 16);
                const int qh = nt * 8 + 2 * tig + c;
                if (qh >= a.G) continue;
                const float inv = 1.f / l;
                float* dst = a.part_o + ((int64_t)it.part_row0 + qh) * D;
#pragma unroll
                for (int mt = 0; mt < KS; ++mt) {
                    dst[mt * 16 + g8] = o[nt][mt][c] * inv;
                    dst[mt * 16 + g8 + 8] = o[nt][mt][c + 2] * inv;
                }
                if (g8 == 0) a.part_lse[it.part_row0 + qh] = (m_run[nt][c] + log2f(l)) * 0.69314718055994531f;
            }
        }
    }

    // never leave with copies in flight (only after a failed wait)
    if (failed && lane == 0)
        for (int s = 0; s < L::kSlots; ++s) {
            volatile int never = 0;
            dev::mbar_wait(&full[s], 0, &never, a.err);
            dev::mbar_wait(&full[s], 1, &never, a.err);
        }
    // the last warp to finish resets the item counter for the next launch
    if (lane == 0) {
        __threadfence();
        const int32_t done = atomicAdd(&a.sched[1], 1);
        if (done == (int32_t)(gridDim.x * kSufWarps) - 1) {
            a.sched[0] = 0;
            a.sched[1] = 0;
            __threadfence();
        }
    }
    // Beside the grouped pass (launched after it with programmatic
    // serialization): end only after it, so that whatever the stream runs
    // next sees both passes' partial rows.
    dev::pdl_wait();
}

// beside: launched right after the grouped pass on the same stream, with
// programmatic serialization.  The grouped pass lets it start as soon as all
// of its CTAs run, so this grid's first CTAs take the SMs the grouped pass
// left free and the rest take each SM the grouped pass gives up, until the
// items run out; every CTA then waits for the grouped pass before it ends.
template <int D, int NT, bool kDevCount = false>
cudaError_t launch_t(const SuffixArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, bool beside,
                     cudaStream_t stream) {
    using L = SufLayout<D>;
    cudaError_t e =
        cudaFuncSetAttribute(k_suffix<D, NT, kDevCount>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::max(1, std::min(sms, (a.n_items + kSufWarps - 1) / kSufWarps));
    if (!beside) {
        k_suffix<D, NT, kDevCount><<<grid, kSufWarps * 32, L::kTotal, stream>>>(a, tk, tv);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kSufWarps * 32);
    cfg.dynamicSmemBytes = L::kTotal;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_suffix<D, NT, kDevCount>, a, tk, tv);
}

SuffixArgs suffix_args(const fca_plan_s* P, const void* q, float scale) {
    SuffixArgs a;
    a.items = P->suffix_items;
    a.n_items = P->hdr.n_suffix_items;
    a.bt = P->bt;
    a.max_blocks = P->max_blocks;
    a.Hq = P->Hq;
    a.G = P->G;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.part_o = P->part_o;
    a.part_lse = P->part_lse;
    a.err = P->dev_status;
    a.sched = P->sched;
    return a;
}

}  // namespace

cudaError_t launch_suffix(const fca_plan_s* P, const void* q, const CUtensorMap& tk, const CUtensorMap& tv,
                          float scale, bool beside, cudaStream_t stream) {
    if (P->async_update) {
        // the item count of the last update is on the device (sched[2]);
        // the grid is sized for the plan's room
        if (P->cap_suffix_items == 0) return cudaSuccess;
        SuffixArgs a = suffix_args(P, q, scale);
        a.n_items = (int32_t)std::min<int64_t>(P->cap_suffix_items, INT32_MAX);
        const bool two = P->G > 8;
        if (P->D == 128)
            return two ? launch_t<128, 2, true>(a, tk, tv, beside, stream)
                       : launch_t<128, 1, true>(a, tk, tv, beside, stream);
        return two ? launch_t<64, 2, true>(a, tk, tv, beside, stream) : launch_t<64, 1, true>(a, tk, tv, beside, stream);
    }
    if (P->hdr.n_suffix_items == 0) return cudaSuccess;
    const SuffixArgs a = suffix_args(P, q, scale);
    const bool two = P->G > 8;
    if (P->D == 128)
        return two ? launch_t<128, 2>(a, tk, tv, beside, stream) : launch_t<128, 1>(a, tk, tv, beside, stream);
    return two ? launch_t<64, 2>(a, tk, tv, beside, stream) : launch_t<64, 1>(a, tk, tv, beside, stream);
}

cudaError_t launch_suffix_devcount(const fca_plan_s* P, const void* q, const CUtensorMap& tk,
                                   const CUtensorMap& tv, float scale, cudaStream_t stream) {
    if (P->hdr.n_suffix_items == 0) return cudaSuccess;
    const SuffixArgs a = suffix_args(P, q, scale);
    const bool two = P->G > 8;
    if (P->D == 128)
        return two ? launch_t<128, 2, true>(a, tk, tv, false, stream)
                   : launch_t<128, 1, true>(a, tk, tv, false, stream);
    return two ? launch_t<64, 2, true>(a, tk, tv, false, stream) : launch_t<64, 1, true>(a, tk, tv, false, stream);
}

}  // namespace fca
