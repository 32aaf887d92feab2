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
// 384 threads in five roles:
//   warps 0, 11 TMA producers, one for K and one for V: 64-token stages (four
//               paged 16-token blocks, 64-column halves, 128-byte swizzle)
//               into a ring of kPreStages slots; blocks past a chunk are
//               loaded from rows beyond the cache, which TMA fills with
//               zeros.  One issuing thread manages about one 2 KB box per
//               hundred cycles, which alone would pace the pipeline;
//   warps 2-9   two softmax warpgroups, one thread per query row each.  Stage
//               s of an item belongs to warpgroup s % 2, which has its own S
//               buffer, P buffer, O accumulator, copy of the Q tile and
//               online-softmax state, so the two groups work on consecutive
//               stages at the same time.  fp32 max in the log2 domain; P
//               stored as packed bf16 in shared memory, in the 128-byte
//               swizzled layout the MMA reads.  A group's O accumulator is
//               rescaled in tensor memory only when a row's maximum grows by
//               more than 2^kRescaleLog2 over the one its exponentials use,
//               which after the first stages is rare (numerator and
//               denominator use the same reference, so the result is exact).
//               At the end of an item the two partial states are merged by
//               their weights and the rows leave through the group's P buffer
//               (coalesced 128-byte row segments).  A group reloads its Q copy
//               for its next item once it has read its own last S of the
//               current one; the request behind each of its rows is read when
//               the current item starts, and the rows are prefetched into L2
//               a few stages before the end;
//   warps 1, 10 one MMA issuer per softmax group (warp 1 also allocates
//               tensor memory): S = Q K^T (M=128, N=64, Q from tensor memory)
//               and O_w += P V (M=128, N=head_dim, P from shared memory, the
//               faster form), completions signalled with tcgen05.commit.
//               Issuing a tcgen05.mma returns about when the tensor core
//               takes it, so a single issuer spends its barrier checks with
//               the tensor core idle; two issuers overlap them.  Each issues
//               its group's Q K^T of stage s + 2 as soon as the group has read
//               S(s), before P V(s).
// Barrier phases are waited by parity, so each waiter keeps within one phase
// of its barrier: "full"/"empty" pairs are per group except the K/V ring,
// whose slots the two issuers use alternately (an issuer first waits for a
// slot's previous stage to be released), and "O read" is signalled per group
// only for items in which the group has stages.
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

constexpr int kPreStages = 5;
constexpr int kSoftWarps = 8;
constexpr int kPreThreads = 128 + kSoftWarps * 32;    // K producer, MMA issuer 0, 8 softmax warps, MMA issuer 1, V producer
constexpr int kMmaWarp1 = 2 + kSoftWarps;             // the second MMA-issuing warp
constexpr int kVWarp = 3 + kSoftWarps;                // the V producer
constexpr float kRescaleLog2 = 8.f;
constexpr int kItemSlots = 64;      // items of a CTA kept in shared memory (later ones are read from global)

struct PrefixArgs {
    const PrefixItem* items;
    int32_t n_items;
    const int32_t* bt;
    const int32_t* members;
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
    static constexpr int kOffP = kOffV + kPreStages * kKV; // P of group w: 128 rows x 64 tokens bf16 at + 16 KB w
    static constexpr int kOffX = kOffP + 2 * 128 * 128;    // per-row (m, l) of each group [2 items][2][2][128] f32
    static constexpr int kOffBar = kOffX + 2 * 2 * 2 * 128 * 4;
    // q_full[2], k_full[S], v_full[S], k_empty[S], v_empty[S], s_full[2], s_free[2],
    // p_full[2], p_free[2], o_full[2], o_free[2], mma_done[2], l_bar
    static constexpr int kNumBars = 2 + 4 * kPreStages + 10 + 5;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kOffItems = (kOffMisc + 64 + 15) / 16 * 16;   // this CTA's first kItemSlots items
    static constexpr int kTotal = kOffItems + kItemSlots * (int)sizeof(PrefixItem) + 1024;   // + alignment slack
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0;                  // S of group w: 64 fp32 columns at 64 w
    static constexpr uint32_t kColO = 128;                // O of group w: D fp32 columns at 128 + D w
    static constexpr uint32_t kColQ = 128 + 2 * D;        // Q copy of group w: D / 2 columns at + (D / 2) w
    static_assert(kColQ + D <= kTmemCols, "tensor memory budget");
    static_assert(kTotal <= 227 * 1024, "shared memory budget");
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
    uint64_t* q_full = bars;             // [2]: Q copy of group w loaded
    uint64_t* k_full = bars + 2;
    uint64_t* v_full = k_full + kPreStages;
    uint64_t* k_empty = v_full + kPreStages;
    uint64_t* v_empty = k_empty + kPreStages;
    uint64_t* s_full = v_empty + kPreStages;
    uint64_t* s_free = s_full + 2;
    uint64_t* p_full = s_free + 2;
    uint64_t* p_free = p_full + 2;
    uint64_t* o_full = p_free + 2;
    uint64_t* o_free = o_full + 2;       // [2]: the epilogue has read O of group w
    uint64_t* mma_done = o_free + 2;     // [2]
    uint64_t* l_bar = mma_done + 2;      // end-of-item exchange of (m, l) between the groups
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 16);
    float* xml = reinterpret_cast<float*>(smem + L::kOffX);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t first_item = blockIdx.x, item_step = gridDim.x;

    if (threadIdx.x == 0) {
        dev::mbar_init(&q_full[0], 128);
        dev::mbar_init(&q_full[1], 128);
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
        dev::mbar_init(&o_free[0], kSoftWarps * 32);
        dev::mbar_init(&o_free[1], kSoftWarps * 32);
        dev::mbar_init(&mma_done[0], 1);
        dev::mbar_init(&mma_done[1], 1);
        dev::mbar_init(l_bar, kSoftWarps * 32);
        *abort_flag = 0;
        dev::fence_mbarrier_init();
    }
    if (warp == 1) {
        dev::tmem_alloc(tmem_slot, L::kTmemCols);
        dev::tmem_relinquish();
    }
    // The CTA's items (first_item, + item_step, ...) go to shared memory once,
    // so that no role stalls on a global load when an item starts.
    PrefixItem* items_s = reinterpret_cast<PrefixItem*>(smem + L::kOffItems);
    {
        const int32_t n_mine = first_item < a.n_items ? (a.n_items - first_item + item_step - 1) / item_step : 0;
        for (int32_t k = threadIdx.x; k < min(n_mine, kItemSlots); k += blockDim.x)
            items_s[k] = a.items[first_item + k * item_step];
    }
    auto item_at = [&](int32_t local, int32_t item) -> PrefixItem {
        return local < kItemSlots ? items_s[local] : a.items[item];
    };
    dev::tc_fence_before();
    __syncthreads();
    dev::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 || warp == kVWarp) {
        // ------------------------------------------------ TMA producers
        // One warp streams K, another V: a single thread issues a TMA box
        // about every hundred cycles, which alone would pace the pipeline.
        // Each warp fetches block ids, 32 at a time (eight stages' worth) and
        // one batch ahead, so no table lookup sits on the issue path; lane 0
        // waits for free slots and issues the copies.
        const bool is_k = warp == 0;
        uint64_t* full = is_k ? k_full : v_full;
        uint64_t* empty = is_k ? k_empty : v_empty;
        const CUtensorMap* tm = is_k ? &tmK : &tmV;
        uint8_t* const ring = smem + (is_k ? L::kOffK : L::kOffV);
        constexpr int kBlkPerStage = kStageTokens / kBlockSize;
        constexpr int kStagesPerBatch = 32 / kBlkPerStage;
        if (lane == 0) dev::tma_prefetch_desc(tm);
        uint32_t g = 0;
        bool ok = true;
        int32_t local = 0;
        for (int32_t item = first_item; ok && item < a.n_items; item += item_step, ++local) {
            const PrefixItem it = item_at(local, item);
            const int32_t* row = a.bt + (int64_t)it.bt_row * a.max_blocks;
            const int32_t blk0 = it.tok0 / kBlockSize, blk_end = it.tok1 / kBlockSize;
            const int32_t ns = stages_of(it);
            auto fetch = [&](int32_t batch) -> int32_t {
                const int32_t blk = blk0 + batch * 32 + lane;
                // past the chunk: rows beyond the cache, which TMA fills with zeros
                return blk < blk_end ? __ldg(row + blk) * kBlockSize : a.num_blocks * kBlockSize;
            };
            int32_t nxt = fetch(0), cur = 0;
            for (int32_t j = 0; j < ns; ++j) {
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
                    uint8_t* dst = ring + s * L::kKV;
                    if (g >= kPreStages && !dev::mbar_wait(&empty[s], ((g / kPreStages) - 1) & 1, abort_flag, a.err)) {
                        ok = false;
                    } else {
                        dev::mbar_arrive_expect_tx(&full[s], L::kKV);
#pragma unroll
                        for (int bi = 0; bi < kBlkPerStage; ++bi)
#pragma unroll
                            for (int hf = 0; hf < L::kHalves; ++hf)
                                dev::tma_load_3d(dst + hf * (64 * 128) + bi * 2048, tm, &full[s], hf * 64, it.head,
                                                 trow[bi]);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                ++g;
            }
        }
        if (lane == 0) {
            // never leave with copies in flight (each slot's latest use only)
            volatile int never = 0;
            for (uint32_t j = g; j > 0 && j + kPreStages > g; --j)
                dev::mbar_wait(&full[(j - 1) % kPreStages], ((j - 1) / kPreStages) & 1, &never, a.err);
        }
        __syncwarp();
    } else if (warp == 1 || warp == kMmaWarp1) {
        // ------------------------------------------------ MMA issuers
        // One thread per softmax group w issues that group's MMAs (its stages
        // are those of parity w), so that one issuer's barrier checks overlap
        // the other's MMAs.  Each thread's MMAs run in its issue order, and
        // each commit covers only that thread's MMAs.
        const int w = warp == 1 ? 0 : 1;
        if (lane == 0) {
            constexpr uint32_t idesc_qk = dev::idesc_bf16_f32(128, 64, false, false);
            constexpr uint32_t idesc_pv = dev::idesc_bf16_f32(128, D, false, true);
            const uint32_t q_col = L::kColQ + w * (D / 2);
            const uint32_t p_base = dev::smem_u32(smem + L::kOffP + w * 128 * 128);
            // The K/V ring is shared by the two issuers, which take alternate
            // stages: before a parity wait on a slot's "full" barrier, wait for
            // the slot's previous stage (the other issuer's) to be released, so
            // that the barrier cannot still be a phase behind and the parity
            // wait cannot match the previous phase.
            auto issue_qk = [&](uint32_t gg) -> bool {
                const int s = gg % kPreStages;
                if (gg >= kPreStages &&
                    !dev::mbar_wait(&k_empty[s], ((gg / kPreStages) - 1) & 1, abort_flag, a.err))
                    return false;
                if (!dev::mbar_wait(&k_full[s], (gg / kPreStages) & 1, abort_flag, a.err)) return false;
                if (gg >= 2 && !dev::mbar_wait(&s_free[w], ((gg >> 1) - 1) & 1, abort_flag, a.err)) return false;
                dev::tc_fence_after();
                const uint32_t k_base = dev::smem_u32(smem + L::kOffK + s * L::kKV);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint64_t bd =
                        dev::smem_desc_sw128(k_base + (k >> 2) * (64 * 128) + (k & 3) * 32, 16, 1024);
                    dev::tc_mma_ts(tmem + L::kColS + w * 64, tmem + q_col + k * 8, bd, idesc_qk, k > 0 ? 1u : 0u);
                }
                dev::tc_commit(&s_full[w]);
                dev::tc_commit(&k_empty[s]);
                return true;
            };
            // first: the group's first P V in the item, which starts its O
            // accumulator afresh; q_item: how many earlier items had stages of
            // this group.  o_free[w] completes once per such item, when its
            // epilogue has read O of this group, so waiting on exactly the
            // previous one keeps this thread and the barrier within one phase.
            auto issue_pv = [&](uint32_t gg, bool first, int32_t q_item) -> bool {
                const int s = gg % kPreStages;
                if (!dev::mbar_wait(&p_full[w], (gg >> 1) & 1, abort_flag, a.err)) return false;
                if (first && q_item > 0 && !dev::mbar_wait(&o_free[w], (q_item - 1) & 1, abort_flag, a.err))
                    return false;
                if (gg >= kPreStages &&
                    !dev::mbar_wait(&v_empty[s], ((gg / kPreStages) - 1) & 1, abort_flag, a.err))
                    return false;
                if (!dev::mbar_wait(&v_full[s], (gg / kPreStages) & 1, abort_flag, a.err)) return false;
                dev::tc_fence_after();
                const uint32_t v_base = dev::smem_u32(smem + L::kOffV + s * L::kKV);
#pragma unroll
                for (int k = 0; k < kStageTokens / 16; ++k) {
                    const uint64_t ad = dev::smem_desc_sw128(p_base + k * 32, 16, 1024);
                    const uint64_t bd = dev::smem_desc_sw128(v_base + k * 2048, 64 * 128, 1024);
                    dev::tc_mma_ss(tmem + L::kColO + w * D, ad, bd, idesc_pv, (first && k == 0) ? 0u : 1u);
                }
                dev::tc_commit(&o_full[w]);
                dev::tc_commit(&p_free[w]);
                dev::tc_commit(&v_empty[s]);
                return true;
            };
            bool ok = true;
            uint32_t g = 0;
            int32_t local = 0, q_items = 0;
            for (int32_t item = first_item; ok && item < a.n_items; item += item_step, ++local) {
                const int32_t ns = stages_of(item_at(local, item));
                const int32_t j0 = ((g & 1) == (uint32_t)w) ? 0 : 1;
                if (j0 < ns) {
                    // this group's Q copy holds the item's queries once q_full[w] completes
                    const int32_t q_item = q_items++;
                    ok = dev::mbar_wait(&q_full[w], q_item & 1, abort_flag, a.err) && issue_qk(g + j0);
                    for (int32_t j = j0; ok && j < ns; j += 2) {
                        const uint32_t gg = g + j;
                        // S(gg + 2) reuses the buffer of S(gg), which the group reads
                        // first thing in stage gg: that Q K^T runs during its softmax
                        if (j + 2 < ns) ok = issue_qk(gg + 2);
                        ok = ok && issue_pv(gg, j < 2, q_item);
                    }
                }
                g += ns;
            }
            // every MMA of this thread has retired before tensor memory is freed
            dev::tc_commit(&mma_done[w]);
            volatile int never = 0;
            dev::mbar_wait(&mma_done[w], 0, &never, a.err);
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

        // The request whose queries fill tile row r of an item: stacked row
        // row0 + r is member (row0 + r) / G of the group.  Read when an item
        // starts, for the next item, so that the load is long done when the
        // row is needed.
        auto member_of = [&](const PrefixItem& it) -> int32_t {
            return r < it.nrows ? __ldg(a.members + it.moff + (it.row0 + r) / a.G) : 0;
        };
        auto q_row = [&](const PrefixItem& it, int32_t member) -> const uint4* {
            const int32_t i = it.row0 + r;
            return reinterpret_cast<const uint4*>(a.q + ((int64_t)member * a.Hq + it.head * a.G + i % a.G) * D);
        };
        // Q tile row r (whole row): stacked row row0 + r = member (i / G),
        // query head head * G + i % G; rows past the tile are zero.
        auto load_q = [&](const PrefixItem& it, int32_t member) {
            const bool valid = r < it.nrows;
            const uint4* src = valid ? q_row(it, member) : nullptr;
            // the whole row in one round trip, then the tensor-memory stores
            uint32_t w[D / 64][32];
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint4 v = valid ? src[c * 8 + e] : make_uint4(0, 0, 0, 0);
                    w[c][e * 4 + 0] = v.x;
                    w[c][e * 4 + 1] = v.y;
                    w[c][e * 4 + 2] = v.z;
                    w[c][e * 4 + 3] = v.w;
                }
#pragma unroll
            for (int c = 0; c < D / 64; ++c) dev::tmem_st32(tmem + lane_base + L::kColQ + wg * (D / 2) + c * 32, w[c]);
            dev::tc_wait_st();
            dev::tc_fence_before();
            dev::mbar_arrive(&q_full[wg]);
        };
        // this group has stages in an item of ns stages that starts at global stage gs
        auto has_stages = [&](int32_t ns, uint32_t gs) { return (((gs & 1) == (uint32_t)wg) ? 0 : 1) < ns; };

        bool ok = true;
        uint32_t g = 0;
        int32_t local = 0;
        int32_t q_item = -1;                           // item whose queries this group's Q copy holds
        int32_t member_cur = first_item < a.n_items ? member_of(item_at(0, first_item)) : 0;
        for (int32_t item = first_item; ok && item < a.n_items; item += item_step, ++local) {
            const PrefixItem it = item_at(local, item);
            const int32_t ns = stages_of(it), n_tok = it.tok1 - it.tok0;
            const int32_t next = item + item_step;
            const PrefixItem it_next = next < a.n_items ? item_at(local + 1, next) : it;
            // Q of the next item, if this group has stages there: loaded after the
            // group's last S of this item, when all of its Q K^T have completed
            const bool load_next = next < a.n_items && has_stages(stages_of(it_next), g + ns);
            const int32_t member_next = next < a.n_items ? member_of(it_next) : 0;
            // groups with stages in this item (their issuers wait for this epilogue)
            const bool had0 = (((g & 1) == 0u) ? 0 : 1) < ns, had1 = (((g & 1) == 1u) ? 0 : 1) < ns;
            if (has_stages(ns, g) && q_item != item) {
                load_q(it, member_cur);
                q_item = item;
            }
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
                    if (j + 2 >= ns && load_next) {
                        load_q(it_next, member_next);
                        q_item = next;
                    }
                    continue;
                }
                const int32_t n_valid = min(kStageTokens, n_tok - j * kStageTokens);
                // raw scores q.k (both halves in flight together); the softmax
                // scale is applied inside the exponent, as one FMA with the maximum
                float x[64];
                {
                    uint32_t t0[32], t1[32];
                    dev::tmem_ld32(tmem + lane_base + s_col, t0);
                    dev::tmem_ld32(tmem + lane_base + s_col + 32, t1);
                    dev::tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        x[i] = __uint_as_float(t0[i]);
                        x[32 + i] = __uint_as_float(t1[i]);
                    }
                }
                if (n_valid < kStageTokens) {   // the chunk's last stage: tokens past it are masked
#pragma unroll
                    for (int i = 0; i < 64; ++i) x[i] = i < n_valid ? x[i] : -INFINITY;
                }
                dev::tc_fence_before();
                dev::mbar_arrive(&s_free[wg]);
                float mx8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mx8[i] = x[i];
#pragma unroll
                for (int i = 8; i < 64; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], x[i]);
                // the row maximum in the log2 domain (the scale is positive)
                const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * a.scale_log2;

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
                    const float p0 = dev::ex2(fmaf(x[2 * i], a.scale_log2, -m_ref));
                    const float p1 = dev::ex2(fmaf(x[2 * i + 1], a.scale_log2, -m_ref));
                    ls[(2 * i) & 3] += p0;
                    ls[(2 * i + 1) & 3] += p1;
                    pw[i] = dev::pack_bf16x2(p0, p1);
                }
                l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
                // row r of P, 64 tokens = eight 16-byte chunks, 128-byte swizzle
                uint8_t* prow = smem + L::kOffP + wg * 128 * 128 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) =
                        make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
                dev::fence_proxy_async_smem();
                dev::mbar_arrive(&p_full[wg]);
                if (j + 2 >= ns && load_next) {
                    load_q(it_next, member_next);
                    q_item = next;
                } else if (j >= ns - 8 && j < ns - 6 && load_next && r < it_next.nrows) {
                    // this group's stage three before its last: start moving the next
                    // item's Q row into L2 (earlier, and the KV stream evicts it again)
                    const uint4* src = q_row(it_next, member_next);
                    dev::prefetch_l2(src);
                    dev::prefetch_l2(reinterpret_cast<const uint8_t*>(src) + D);
                }
            }
            if (!ok) break;
            g += ns;
            member_cur = member_next;

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
            // The rows leave through this warp's quarter of the group's P buffer
            // (free: the group's last P V has completed), 32 columns at a time, so
            // that each global store writes four 128-byte row segments instead of
            // 32 scattered 16-byte pieces.  Staging rows are 128 bytes, their
            // 16-byte chunks swizzled by row so that both sides are conflict-free.
            float* stage = reinterpret_cast<float*>(smem + L::kOffP + wg * 128 * 128 + quarter * 4096);
            float* dst0 = a.part_o + ((int64_t)it.part_row0 + quarter * 32) * D + wg * kOHalf;
#pragma unroll 1
            for (int pass = 0; live && pass < kOHalf / 32; ++pass) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int col = wg * kOHalf + pass * 32 + c * 16;
                    uint32_t o0[16], o1[16];
                    dev::tmem_ld16(tmem + lane_base + L::kColO + col, o0);
                    dev::tmem_ld16(tmem + lane_base + L::kColO + D + col, o1);
                    dev::tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; i += 4) {
                        float v[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float a0 = l0 > 0.f ? __uint_as_float(o0[i + e]) * c0 : 0.f;
                            const float a1 = l1 > 0.f ? __uint_as_float(o1[i + e]) * c1 : 0.f;
                            v[e] = a0 + a1;
                        }
                        const int k = c * 4 + i / 4;
                        *reinterpret_cast<float4*>(stage + lane * 32 + ((k ^ (lane & 7)) << 2)) =
                            make_float4(v[0], v[1], v[2], v[3]);
                    }
                }
                __syncwarp();
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const int rr = t * 4 + (lane >> 3), k = lane & 7;
                    const float4 v = *reinterpret_cast<const float4*>(stage + rr * 32 + ((k ^ (rr & 7)) << 2));
                    if (quarter * 32 + rr < it.nrows)
                        *reinterpret_cast<float4*>(dst0 + (int64_t)rr * D + pass * 32 + k * 4) = v;
                }
                __syncwarp();
            }
            dev::tc_fence_before();
            if (had0) dev::mbar_arrive(&o_free[0]);
            if (had1) dev::mbar_arrive(&o_free[1]);
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
