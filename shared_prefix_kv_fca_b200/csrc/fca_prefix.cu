// Grouped pass over a group's shared prefix blocks on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// "ZoRRo Inference & Forest Cascade Attention", "Core Mechanism" step 2,
// first bullet: one grouped pass over the shared prefix blocks, so that each
// block is read once per group instead of once per request.  All queries of a
// group that read the same KV head -- members x G query heads -- are stacked
// into one 128-row Q tile, which turns the pass into a dense contraction
// against the shared K and V.
//
// Work item = (group, KV head, 128-row Q tile, token chunk).  The kernel is
// persistent: one CTA per SM walks its items (blockIdx.x, +gridDim.x, ...),
// tensor memory is allocated once, and the K/V stream runs on across items.
// 320 threads in three roles:
//   warp 0      TMA producer: 64-token stages of K and V (four paged 16-token
//               blocks, 64-column halves, 128-byte swizzle) into a ring of
//               kPreStages slots; blocks past a chunk are loaded from rows
//               beyond the cache, which TMA fills with zeros;
//   warp 1      allocates tensor memory and, from one thread, issues
//               S = Q K^T (M=128, N=64) and O_w += P V (M=128, N=head_dim),
//               signalling completions with tcgen05.commit.  Q and P are the
//               A operands and live in tensor memory next to S and O, so all
//               of shared memory holds the K/V ring (the stages a slow HBM
//               stream needs in flight); a K slot is released as soon as its
//               Q K^T has run, a V slot after its P V;
//   warps 2-9   two softmax warpgroups, one thread per query row each.  Stage
//               s of an item belongs to warpgroup s % 2, which has its own S
//               buffer, P buffer, O accumulator and online-softmax state, so
//               the two groups work on consecutive stages at the same time
//               and never wait for each other inside an item.  fp32 max in
//               the log2 domain; P stored to tensor memory as packed bf16.  A group's O accumulator is rescaled in
//               tensor memory only when a row's maximum grows by more than
//               2^kRescaleLog2 over the one its exponentials use, which after
//               the first stages is rare (numerator and denominator use the
//               same reference, so the result is exact).  At the end of an
//               item the two partial states are merged by their weights.
// Warps whose 32 tile rows are all past the group's stacked rows skip the
// softmax and the output, and keep only the barrier protocol.
// Output: one partial row (normalised o, natural-log lse) per stacked query
// row, merged later with the row's other partials.
#include <algorithm>

#include <cuda_bf16.h>

#include "fca_device.cuh"
#include "fca_internal.h"

namespace fca {

namespace {

constexpr int kPreStages = 6;
constexpr int kSoftWarps = 8;
constexpr int kPreThreads = 64 + kSoftWarps * 32;
constexpr float kRescaleLog2 = 8.f;

struct PrefixArgs {
    const PrefixItem* items;
    int32_t n_items;
    const int32_t* bt;
    const int32_t* members;
    const int32_t* g_moff;
    int32_t max_blocks, num_blocks, Hq, G;
    const __nv_bfloat16* q;
    float scale_log2;
    float* part_o;
    float* part_lse;
    int32_t* err;
};

template <int D>
struct PreLayout {
    static constexpr int kHalves = D / 64;
    static constexpr int kKV = kHalves * 64 * 128;        // one 64-token K (or V) stage
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kPreStages * kKV;
    static constexpr int kOffX = kOffV + kPreStages * kKV; // per-row (m, l) of each group [2 items][2][2][128] f32
    static constexpr int kOffBar = kOffX + 2 * 2 * 2 * 128 * 4;
    // q_full, k_full[S], v_full[S], k_empty[S], v_empty[S], s_full[2], s_free[2],
    // p_full[2], p_free[2], o_full[2], o_free, mma_done, l_bar
    static constexpr int kNumBars = 1 + 4 * kPreStages + 10 + 3;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kTotal = kOffMisc + 64 + 1024;   // + alignment slack
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0;                  // S of group w: 64 fp32 columns at 64 w
    static constexpr uint32_t kColO = 128;                // O of group w: D fp32 columns at 128 + D w
    static constexpr uint32_t kColP = 128 + 2 * D;        // P of group w: 32 columns (64 bf16) at + 32 w
    static constexpr uint32_t kColQ = kColP + 64;         // Q: D / 2 columns (D bf16)
    static_assert(kColQ + D / 2 <= kTmemCols, "tensor memory budget");
};

__device__ __forceinline__ int32_t stages_of(const PrefixItem& it) {
    return (it.tok1 - it.tok0 + kStageTokens - 1) / kStageTokens;
}

template <int D>
__global__ void __launch_bounds__(kPreThreads, 1)
    k_prefix(PrefixArgs a, const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
    using L = PreLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* v_full = k_full + kPreStages;
    uint64_t* k_empty = v_full + kPreStages;
    uint64_t* v_empty = k_empty + kPreStages;
    uint64_t* s_full = v_empty + kPreStages;
    uint64_t* s_free = s_full + 2;
    uint64_t* p_full = s_free + 2;
    uint64_t* p_free = p_full + 2;
    uint64_t* o_full = p_free + 2;
    uint64_t* o_free = o_full + 2;
    uint64_t* mma_done = o_free + 1;
    uint64_t* l_bar = mma_done + 1;      // end-of-item exchange of (m, l) between the groups
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 16);
    float* xml = reinterpret_cast<float*>(smem + L::kOffX);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t first_item = blockIdx.x, item_step = gridDim.x;

    if (threadIdx.x == 0) {
        dev::mbar_init(q_full, 128);
        for (int st = 0; st < kPreStages; ++st) {
            dev::mbar_init(&k_full[st], 1);
            dev::mbar_init(&v_full[st], 1);
            dev::mbar_init(&k_empty[st], 1);
            dev::mbar_init(&v_empty[st], 1);
        }
        for (int b = 0; b < 2; ++b) {
            dev::mbar_init(&s_full[b], 1);
            dev::mbar_init(&s_free[b], 128);
            dev::mbar_init(&p_full[b], 128);
            dev::mbar_init(&p_free[b], 1);
            dev::mbar_init(&o_full[b], 1);
        }
        dev::mbar_init(o_free, kSoftWarps * 32);
        dev::mbar_init(mma_done, 1);
        dev::mbar_init(l_bar, kSoftWarps * 32);
        *abort_flag = 0;
        dev::fence_mbarrier_init();
    }
    if (warp == 1) {
        dev::tmem_alloc(tmem_slot, L::kTmemCols);
        dev::tmem_relinquish();
    }
    dev::tc_fence_before();
    __syncthreads();
    dev::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        // The whole warp fetches block ids, 32 at a time (eight stages' worth)
        // and one batch ahead, so no table lookup sits on the issue path;
        // lane 0 waits for free slots and issues the copies.
        constexpr int kBlkPerStage = kStageTokens / kBlockSize;
        constexpr int kStagesPerBatch = 32 / kBlkPerStage;
        if (lane == 0) {
            dev::tma_prefetch_desc(&tmK);
            dev::tma_prefetch_desc(&tmV);
        }
        uint32_t g = 0;
        bool ok = true;
        int32_t pending_k = -1;     // stage whose K copies are in flight but whose V is not issued
        for (int32_t item = first_item; ok && item < a.n_items; item += item_step) {
            const PrefixItem it = a.items[item];
            const int32_t* row = a.bt + (int64_t)it.bt_row * a.max_blocks;
            const int32_t blk0 = it.tok0 / kBlockSize, blk_end = it.tok1 / kBlockSize;
            const int32_t ns = stages_of(it);
            auto fetch = [&](int32_t batch) -> int32_t {
                const int32_t blk = blk0 + batch * 32 + lane;
                // past the chunk: rows beyond the cache, which TMA fills with zeros
                return blk < blk_end ? __ldg(row + blk) * kBlockSize : a.num_blocks * kBlockSize;
            };
            int32_t nxt = fetch(0), cur = 0;
            for (int32_t j = 0; j < ns; ++j, ++g) {
                if (j % kStagesPerBatch == 0) {
                    cur = nxt;
                    nxt = fetch(j / kStagesPerBatch + 1);
                }
                int32_t trow[kBlkPerStage];
#pragma unroll
                for (int bi = 0; bi < kBlkPerStage; ++bi)
                    trow[bi] = __shfl_sync(0xffffffffu, cur, (j % kStagesPerBatch) * kBlkPerStage + bi);
                if (lane == 0) {
                    const int s = g % kPreStages;
                    const uint32_t ph = ((g / kPreStages) - 1) & 1;
                    uint8_t* kdst = smem + L::kOffK + s * L::kKV;
                    uint8_t* vdst = smem + L::kOffV + s * L::kKV;
                    if (g >= kPreStages && !dev::mbar_wait(&k_empty[s], ph, abort_flag, a.err)) {
                        ok = false;
                    } else {
                        dev::mbar_arrive_expect_tx(&k_full[s], L::kKV);
#pragma unroll
                        for (int bi = 0; bi < kBlkPerStage; ++bi)
#pragma unroll
                            for (int hf = 0; hf < L::kHalves; ++hf)
                                dev::tma_load_3d(kdst + hf * (64 * 128) + bi * 2048, &tmK, &k_full[s], hf * 64,
                                                 it.head, trow[bi]);
                        pending_k = (int32_t)g;
                        if (g >= kPreStages && !dev::mbar_wait(&v_empty[s], ph, abort_flag, a.err)) {
                            ok = false;
                        } else {
                            dev::mbar_arrive_expect_tx(&v_full[s], L::kKV);
#pragma unroll
                            for (int bi = 0; bi < kBlkPerStage; ++bi)
#pragma unroll
                                for (int hf = 0; hf < L::kHalves; ++hf)
                                    dev::tma_load_3d(vdst + hf * (64 * 128) + bi * 2048, &tmV, &v_full[s], hf * 64,
                                                     it.head, trow[bi]);
                            pending_k = -1;
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
        if (lane == 0) {
            // never leave with copies in flight
            volatile int never = 0;
            if (pending_k >= 0)
                dev::mbar_wait(&k_full[pending_k % kPreStages], (pending_k / kPreStages) & 1, &never, a.err);
            for (uint32_t j = g; j > 0 && j + kPreStages > g; --j) {
                dev::mbar_wait(&k_full[(j - 1) % kPreStages], ((j - 1) / kPreStages) & 1, &never, a.err);
                dev::mbar_wait(&v_full[(j - 1) % kPreStages], ((j - 1) / kPreStages) & 1, &never, a.err);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = dev::idesc_bf16_f32(128, 64, false, false);
            constexpr uint32_t idesc_pv = dev::idesc_bf16_f32(128, D, false, true);
            auto issue_qk = [&](uint32_t gg) -> bool {
                const int s = gg % kPreStages, sb = gg & 1;
                if (!dev::mbar_wait(&k_full[s], (gg / kPreStages) & 1, abort_flag, a.err)) return false;
                if (gg >= 2 && !dev::mbar_wait(&s_free[sb], ((gg >> 1) - 1) & 1, abort_flag, a.err)) return false;
                dev::tc_fence_after();
                const uint32_t k_base = dev::smem_u32(smem + L::kOffK + s * L::kKV);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint64_t bd =
                        dev::smem_desc_sw128(k_base + (k >> 2) * (64 * 128) + (k & 3) * 32, 16, 1024);
                    dev::tc_mma_ts(tmem + L::kColS + sb * 64, tmem + L::kColQ + k * 8, bd, idesc_qk, k > 0 ? 1u : 0u);
                }
                dev::tc_commit(&s_full[sb]);
                dev::tc_commit(&k_empty[s]);
                return true;
            };
            // first: the first P V of group (gg & 1) in this item, which starts
            // its O accumulator afresh once the previous item's epilogue read it
            auto issue_pv = [&](uint32_t gg, bool first, int32_t local_item) -> bool {
                const int s = gg % kPreStages, pb = gg & 1;
                if (!dev::mbar_wait(&p_full[pb], (gg >> 1) & 1, abort_flag, a.err)) return false;
                if (first && local_item > 0 && !dev::mbar_wait(o_free, (local_item - 1) & 1, abort_flag, a.err))
                    return false;
                if (!dev::mbar_wait(&v_full[s], (gg / kPreStages) & 1, abort_flag, a.err)) return false;
                dev::tc_fence_after();
                const uint32_t v_base = dev::smem_u32(smem + L::kOffV + s * L::kKV);
#pragma unroll
                for (int k = 0; k < kStageTokens / 16; ++k) {
                    const uint64_t bd = dev::smem_desc_sw128(v_base + k * 2048, 64 * 128, 1024);
                    dev::tc_mma_ts(tmem + L::kColO + pb * D, tmem + L::kColP + pb * 32 + k * 8, bd, idesc_pv,
                                   (first && k == 0) ? 0u : 1u);
                }
                dev::tc_commit(&o_full[pb]);
                dev::tc_commit(&p_free[pb]);
                dev::tc_commit(&v_empty[s]);
                return true;
            };
            bool ok = true;
            uint32_t g = 0;
            int32_t local = 0;
            if (first_item < a.n_items) ok = dev::mbar_wait(q_full, 0, abort_flag, a.err) && issue_qk(0);
            for (int32_t item = first_item; ok && item < a.n_items; item += item_step, ++local) {
                const int32_t ns = stages_of(a.items[item]);
                const bool has_next = item + item_step < a.n_items;
                for (int32_t j = 0; ok && j < ns; ++j) {
                    const uint32_t gg = g + j;
                    if (j + 1 < ns) {
                        ok = issue_qk(gg + 1) && issue_pv(gg, j < 2, local);
                    } else {
                        // last stage: finish this item's O first, then start the next item
                        ok = issue_pv(gg, j < 2, local);
                        if (ok && has_next)
                            ok = dev::mbar_wait(q_full, (local + 1) & 1, abort_flag, a.err) && issue_qk(gg + 1);
                    }
                }
                g += ns;
            }
            // every MMA of this thread has retired before tensor memory is freed
            dev::tc_commit(mma_done);
            volatile int never = 0;
            dev::mbar_wait(mma_done, 0, &never, a.err);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax warpgroups
        const int quarter = warp & 3;                  // TMEM lane quarter of this warp
        const int wg = (warp - 2) >> 2;                // stages of parity wg are this group's
        const int r = quarter * 32 + lane;             // tile row
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_col = L::kColS + wg * 64, o_col = L::kColO + wg * D;
        constexpr int kOHalf = D / 2;

        // Q tile row r (whole row): stacked row row0 + r = member (i / G),
        // query head head * G + i % G; rows past the tile are zero.
        auto load_q = [&](const PrefixItem& it) {
            const bool valid = r < it.nrows;
            const uint4* src = nullptr;
            if (valid) {
                const int32_t i = it.row0 + r;
                const int32_t member = a.members[a.g_moff[it.group] + i / a.G];
                src = reinterpret_cast<const uint4*>(a.q + ((int64_t)member * a.Hq + it.head * a.G + i % a.G) * D);
            }
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                uint32_t w[32];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint4 v = valid ? src[c * 8 + e] : make_uint4(0, 0, 0, 0);
                    w[e * 4 + 0] = v.x;
                    w[e * 4 + 1] = v.y;
                    w[e * 4 + 2] = v.z;
                    w[e * 4 + 3] = v.w;
                }
                dev::tmem_st32(tmem + lane_base + L::kColQ + c * 32, w);
            }
            dev::tc_wait_st();
            dev::tc_fence_before();
            dev::mbar_arrive(q_full);
        };

        bool ok = true;
        uint32_t g = 0;
        int32_t local = 0;
        if (wg == 0 && first_item < a.n_items) load_q(a.items[first_item]);
        for (int32_t item = first_item; ok && item < a.n_items; item += item_step, ++local) {
            const PrefixItem it = a.items[item];
            const int32_t ns = stages_of(it), n_tok = it.tok1 - it.tok0;
            const bool has_next = item + item_step < a.n_items;
            float m_ref = -INFINITY, l_run = 0.f;
            int32_t my_last = -1;                      // my last stage of this item (global index)
            // A warp whose 32 tile rows are all past the group's stacked rows has
            // nothing to compute: it skips the softmax and the output, and keeps
            // only the barrier protocol (its P and O rows are never read back).
            const bool live = quarter * 32 < it.nrows;
            for (int32_t j = ((g & 1) == (uint32_t)wg) ? 0 : 1; j < ns; j += 2) {
                const uint32_t gg = g + j;
                my_last = (int32_t)gg;
                bool got = dev::mbar_wait(&s_full[wg], (gg >> 1) & 1, abort_flag, a.err);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                dev::tc_fence_after();
                if (!live) {
                    // same arrivals in the same order as a live warp; p_free first,
                    // so that this arrival cannot count towards an earlier phase
                    dev::mbar_arrive(&s_free[wg]);
                    if (gg >= 2) {
                        got = dev::mbar_wait(&p_free[wg], ((gg >> 1) - 1) & 1, abort_flag, a.err);
                        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                    }
                    dev::mbar_arrive(&p_full[wg]);
                    if (j + 1 == ns && has_next) load_q(a.items[item + item_step]);
                    continue;
                }
                const int32_t n_valid = min(kStageTokens, n_tok - j * kStageTokens);
                float x[64];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t t[32];
                    dev::tmem_ld32(tmem + lane_base + s_col + h2 * 32, t);
                    dev::tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        x[h2 * 32 + i] = h2 * 32 + i < n_valid ? __uint_as_float(t[i]) * a.scale_log2 : -INFINITY;
                }
                dev::tc_fence_before();
                dev::mbar_arrive(&s_free[wg]);
                float mx8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mx8[i] = x[i];
#pragma unroll
                for (int i = 8; i < 64; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], x[i]);
                const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));

                float alpha = 1.f;
                bool rescale = false;
                if (m_ref == -INFINITY) {
                    m_ref = mx;                       // this group's first stage of the item
                } else if (mx > m_ref + kRescaleLog2) {
                    alpha = dev::ex2(m_ref - mx);
                    m_ref = mx;
                    rescale = true;
                }
                l_run *= alpha;
                if (__any_sync(0xffffffffu, rescale)) {
                    // the accumulator may be touched only after this group's previous P V retired
                    got = dev::mbar_wait(&o_full[wg], ((gg >> 1) - 1) & 1, abort_flag, a.err);
                    if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                    dev::tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < D / 16; ++c) {
                        uint32_t ov[16];
                        const uint32_t ta = tmem + lane_base + o_col + c * 16;
                        dev::tmem_ld16(ta, ov);
                        dev::tc_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                        dev::tmem_st16(ta, ov);
                    }
                    dev::tc_wait_st();
                    dev::tc_fence_before();
                }
                if (gg >= 2) {
                    got = dev::mbar_wait(&p_free[wg], ((gg >> 1) - 1) & 1, abort_flag, a.err);
                    if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                }
                float ls[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t pw[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float p0 = dev::ex2(x[2 * i] - m_ref), p1 = dev::ex2(x[2 * i + 1] - m_ref);
                    ls[(2 * i) & 3] += p0;
                    ls[(2 * i + 1) & 3] += p1;
                    pw[i] = dev::pack_bf16x2(p0, p1);
                }
                l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
                dev::tmem_st32(tmem + lane_base + L::kColP + wg * 32, pw);
                dev::tc_wait_st();
                dev::tc_fence_before();
                dev::mbar_arrive(&p_full[wg]);
                // the group that read the item's last S knows every Q K^T of the
                // item has completed: it refills the Q tile for the next item
                if (j + 1 == ns && has_next) load_q(a.items[item + item_step]);
            }
            if (!ok) break;
            g += ns;

            // epilogue: wait for this group's last P V, swap (m, l) with the other
            // group, and write half of the columns of the merged, normalised rows
            if (my_last >= 0) {
                bool got = dev::mbar_wait(&o_full[wg], ((uint32_t)my_last >> 1) & 1, abort_flag, a.err);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            }
            // (double-buffered by item: the other group may already be writing the next item's)
            float* xb = xml + (local & 1) * 512;
            xb[(wg * 2 + 0) * 128 + r] = m_ref;
            xb[(wg * 2 + 1) * 128 + r] = l_run;
            dev::mbar_arrive(l_bar);
            {
                bool got = dev::mbar_wait(l_bar, local & 1, abort_flag, a.err);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            }
            dev::tc_fence_after();
            const float m0 = xb[0 * 128 + r], l0 = xb[1 * 128 + r];
            const float m1 = xb[2 * 128 + r], l1 = xb[3 * 128 + r];
            const float m = fmaxf(m0, m1);
            const float w0 = l0 > 0.f ? dev::ex2(m0 - m) : 0.f, w1 = l1 > 0.f ? dev::ex2(m1 - m) : 0.f;
            const float l_tot = l0 * w0 + l1 * w1;
            const float inv = 1.f / l_tot, c0 = w0 * inv, c1 = w1 * inv;
            const bool row_valid = r < it.nrows;
            float* dst = a.part_o + ((int64_t)it.part_row0 + r) * D + wg * kOHalf;
#pragma unroll
            for (int c = 0; live && c < kOHalf / 16; ++c) {
                uint32_t o0[16], o1[16];
                dev::tmem_ld16(tmem + lane_base + L::kColO + wg * kOHalf + c * 16, o0);
                dev::tmem_ld16(tmem + lane_base + L::kColO + D + wg * kOHalf + c * 16, o1);
                dev::tc_wait_ld();
                if (row_valid) {
#pragma unroll
                    for (int i = 0; i < 16; i += 4) {
                        float v[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float a0 = l0 > 0.f ? __uint_as_float(o0[i + e]) * c0 : 0.f;
                            const float a1 = l1 > 0.f ? __uint_as_float(o1[i + e]) * c1 : 0.f;
                            v[e] = a0 + a1;
                        }
                        *reinterpret_cast<float4*>(dst + c * 16 + i) = make_float4(v[0], v[1], v[2], v[3]);
                    }
                }
            }
            dev::tc_fence_before();
            dev::mbar_arrive(o_free);
            if (wg == 0 && row_valid)
                a.part_lse[it.part_row0 + r] = (m + __log2f(l_tot)) * 0.69314718055994531f;
        }
    }

    dev::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        dev::tc_fence_after();
        dev::tmem_dealloc(tmem, L::kTmemCols);
    }
}

template <int D>
cudaError_t launch_prefix_t(const PrefixArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, int max_ctas,
                            cudaStream_t stream) {
    using L = PreLayout<D>;
    cudaError_t e = cudaFuncSetAttribute(k_prefix<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (max_ctas > 0) sms = std::min(sms, max_ctas);
    const int grid = std::max(1, std::min(sms, a.n_items));
    k_prefix<D><<<grid, kPreThreads, L::kTotal, stream>>>(a, tk, tv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefix(const fca_plan_s* P, const void* q, const CUtensorMap& tk, const CUtensorMap& tv,
                          float scale, int max_ctas, cudaStream_t stream) {
    const int n = P->hdr.n_prefix_items;
    if (n == 0) return cudaSuccess;
    PrefixArgs a;
    a.items = P->prefix_items;
    a.n_items = n;
    a.bt = P->bt;
    a.members = P->members;
    a.g_moff = P->g_moff;
    a.max_blocks = P->max_blocks;
    a.num_blocks = P->num_blocks;
    a.Hq = P->Hq;
    a.G = P->G;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.part_o = P->part_o;
    a.part_lse = P->part_lse;
    a.err = P->dev_status;
    if (P->D == 128) return launch_prefix_t<128>(a, tk, tv, max_ctas, stream);
    return launch_prefix_t<64>(a, tk, tv, max_ctas, stream);
}

}  // namespace fca
