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
// and every role runs on across item boundaries, so an item change costs no
// pipeline drain: the next item's Q tile is written while the current one
// streams, and a finished item's output is drained from its accumulator
// while the next item accumulates into the other one.  Pipeline stage = 128
// tokens (eight paged blocks).
//
// 384 threads in five roles (warps 4-7 and 8-11 are whole warpgroups, so
// that each reaches all 128 tensor-memory lanes):
//   warps 0, 2   TMA producers, one for K and one for V, each into its own
//                ring of 128-token slots (K is consumed a stage before V, so
//                each ring's depth is its own lead); eight lanes issue one
//                block's boxes each.  Blocks past a chunk are loaded from rows
//                beyond the cache, which TMA fills with zeros;
//   warps 1, 3   MMA issuers, one thread each (warp 1 also allocates tensor
//                memory): warp 1 issues S = Q K^T (M 128, N 128; Q and K in
//                shared memory) into one of two S buffers, so that the Q K^T
//                of a stage runs during the softmax of the one before; warp 3
//                issues O += P V with P read from tensor memory, where the
//                softmax wrote it over the S it came from, and V from shared
//                memory, into the item's O buffer (two, alternating by item);
//   warps 4-7    softmax: one thread per tile row (tensor-memory lane).  Online
//                softmax in the log2 domain; the O accumulator is rescaled in
//                tensor memory only when a row's maximum grows by more than
//                2^kRescaleLog2 over the reference its exponentials use (rare
//                after the first stage; numerator and denominator share the
//                reference, so the result is exact).  Two row sums: of the
//                bf16-rounded P, the weights P V actually applies (o is
//                normalised by it, so that it stays a weighted mean of V), and
//                of the unrounded values (for the lse);
//   warps 8-11   Q tile loader and epilogue: hold the next item's query rows
//                in registers (loaded an item ahead), write them into the Q
//                tile once the current item's last Q K^T has completed, and
//                turn a finished item's accumulator into normalised partial
//                rows (o, natural-log lse): through a shared-memory staging
//                buffer, so that every global store writes whole 128-byte
//                lines.
// Groups of at most 64 stacked rows fill the tile twice: tile rows j and
// j + 16 of each 32-row quarter hold the same query row.  Tensor-memory
// accesses of two 16-lane halves (.16x32bx2) give threads j and j + 16 of a
// warp lane j's columns [c, c + n) and [c + 64, c + 64 + n): each takes half
// the row's tokens, they write the two halves of lane j's P, so lane j's O is
// the whole row's and lanes 16-31 are never read.  All four SM
// sub-partitions share the softmax, half a row per thread.
// Every wait is bounded (fca_device.cuh); a role that gives up sets the CTA's
// abort flag, the others leave at their next wait, in-flight copies and MMAs
// are drained, and tensor memory is freed.  Barrier phases are waited by
// parity, and the protocol keeps each waiter within one phase of its barrier.
#include <algorithm>

#include <cuda_bf16.h>

#include "fca_device.cuh"
#include "fca_internal.h"

namespace fca {

namespace {

constexpr int kStage = kStageTokens;                // tokens per pipeline stage
constexpr int kBlkPerStage = kStage / kBlockSize;   // paged blocks per stage
constexpr int kThreads = 384;
constexpr int kVWarp = 2;                           // the V producer
constexpr int kPVWarp = 3;                          // the P V issuer
constexpr int kSoftWarp0 = 4;                       // first softmax warp
constexpr int kEpiWarp0 = 8;                        // first loader / epilogue warp
constexpr float kRescaleLog2 = 8.f;
constexpr float kRedoLog2 = 64.f;

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
    static constexpr int kHalves = D / 64;              // 64-element (128-byte) swizzle atoms per row
    static constexpr int kQBytes = 128 * D * 2;         // Q tile: 128 rows, K-major
    static constexpr int kStageBytes = 4 * 32 * 128;    // epilogue staging: 4 warps x 32 rows x 128 B
    static constexpr int kKV = kStage * D * 2;          // one K or V stage
    static constexpr int kKSlots = D == 128 ? 3 : 4;    // K ring
    static constexpr int kVSlots = D == 128 ? 2 : 4;    // V ring
    static constexpr int kOffQ = 0;
    static constexpr int kOffStg = kOffQ + kQBytes;
    static constexpr int kOffK = kOffStg + 2 * kStageBytes;   // two staging buffers
    static constexpr int kOffV = kOffK + kKSlots * kKV;
    static constexpr int kOffML = kOffV + kVSlots * kKV;   // [3][128] f32: an item's row m, l exact, l rounded
    static constexpr int kOffBar = kOffML + 3 * 128 * 4;
    static constexpr int kNumBars = 2 * (kKSlots + kVSlots) + 17;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kBytes = kOffMisc + 32;
    static constexpr int kAlloc = kBytes + 1024;        // the operands want 1024-byte alignment
    static constexpr uint32_t kColS = 0;                // S / P buffer b: 128 fp32 columns at 128 b
    static constexpr uint32_t kColO = 256;              // O buffer b: D fp32 columns at 256 + D b
    static constexpr uint32_t kTmemCols = 512;
    static_assert(kColO + 2 * D <= kTmemCols, "tensor memory budget");
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ int32_t stages_of(const PrefixItem& it) {
    return (it.tok1 - it.tok0 + kStage - 1) / kStage;
}

__device__ __forceinline__ PrefixItem load_item(const PrefixItem* items, int32_t i) {
    const int4* p = reinterpret_cast<const int4*>(items + i);
    const int4 a = __ldg(p), b = __ldg(p + 1);
    PrefixItem it;
    it.moff = a.x;
    it.head = a.y;
    it.row0 = a.z;
    it.nrows = a.w;
    it.tok0 = b.x;
    it.tok1 = b.y;
    it.bt_row = b.z;
    it.part_row0 = b.w;
    return it;
}

// The items of this CTA (blockIdx.x, + gridDim.x, ...) in order, each record
// read one item ahead so that no role waits for a global load when an item
// starts.
struct ItemCursor {
    const PrefixItem* items;
    int32_t first, step, n_mine, li;
    PrefixItem cur, nxt;
    __device__ __forceinline__ ItemCursor(const PrefixItem* it, int32_t f, int32_t s, int32_t n)
        : items(it), first(f), step(s), n_mine(n), li(0) {
        if (n > 0) cur = load_item(items, f);
        if (n > 1) nxt = load_item(items, f + s);
    }
    __device__ __forceinline__ bool has_next() const { return li + 1 < n_mine; }
    __device__ __forceinline__ void advance() {
        ++li;
        cur = nxt;
        if (li + 1 < n_mine) nxt = load_item(items, first + (li + 1) * step);
    }
};

// Tile row t of an item holds stacked row real_row(t) (>= nrows: padding).
// With at most 64 rows the tile holds each row twice (lanes j and j + 16 of a
// 32-lane quarter).
__device__ __forceinline__ bool dup_of(const PrefixItem& it) { return it.nrows <= 64; }
__device__ __forceinline__ int32_t real_row(int t, bool dup) { return dup ? (t >> 5) * 16 + (t & 15) : t; }

// Byte offset of 16-byte chunk c (< 8) of row r in 64-element atom `atom` of
// a K-major, 128-byte swizzled tile whose atoms are `atom_bytes` apart.
__device__ __forceinline__ uint32_t sw128_off(int r, int atom, int c, int atom_bytes) {
    return atom * atom_bytes + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4);
}

// Round r (0, 1) of a softmax thread's columns of an S buffer (raw scores
// q.k), masked from column n_valid on when MASK: 64 columns of the row, or,
// for a duplicated row, 32 of this thread's half.
template <bool DUP, bool MASK>
__device__ __forceinline__ void s_round(uint32_t s_addr, int r, int copy, int n_valid, float (&xc)[DUP ? 32 : 64]) {
    if (!DUP) {
        uint32_t r0[32], r1[32];
        dev::tmem_ld32(s_addr + 64 * r, r0);
        dev::tmem_ld32(s_addr + 64 * r + 32, r1);
        dev::tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            xc[i] = (!MASK || 64 * r + i < n_valid) ? __uint_as_float(r0[i]) : -INFINITY;
            xc[(DUP ? 0 : 32) + i] = (!MASK || 64 * r + 32 + i < n_valid) ? __uint_as_float(r1[i]) : -INFINITY;
        }
    } else {
        uint32_t r0[32];
        dev::tmem_ld16x2_x32<64>(s_addr + 32 * r, r0);
        dev::tc_wait_ld();
        const int c0 = copy * 64 + 32 * r;
#pragma unroll
        for (int i = 0; i < 32; ++i) xc[i] = (!MASK || c0 + i < n_valid) ? __uint_as_float(r0[i]) : -INFINITY;
    }
}

// Row maximum of a stage's S (raw scores), over both halves of a duplicated row.
template <bool DUP, bool MASK>
__device__ __forceinline__ float s_rowmax(uint32_t s_addr, int copy, int n_valid) {
    float mx = -INFINITY;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        float xc[DUP ? 32 : 64];
        s_round<DUP, MASK>(s_addr, r, copy, n_valid, xc);
#pragma unroll
        for (int i = 0; i < (DUP ? 32 : 64); i += 2) mx = dev::max3(mx, xc[i], xc[i + 1]);
    }
    if (DUP) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    return mx;
}

// P of a stage against the reference m_ref (log2 domain): packed bf16 pairs
// in pw, the sum of the values (se) and of their bf16 roundings (sr).
// Returns the stage's row maximum in the log2 domain.
template <bool DUP, bool MASK>
__device__ __forceinline__ float s_exps(uint32_t s_addr, int copy, int n_valid, float scale_log2, float m_ref,
                                        uint32_t (&pw)[kStage / 2], float& se, float& sr) {
    constexpr int kPer = DUP ? 32 : 64;
    float2 e = make_float2(0.f, 0.f), q = make_float2(0.f, 0.f);
    float mx = -INFINITY;
    const float2 sc = make_float2(scale_log2, scale_log2), nm = make_float2(-m_ref, -m_ref);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        float xc[kPer];
        s_round<DUP, MASK>(s_addr, r, copy, n_valid, xc);
#pragma unroll
        for (int i = 0; i < kPer; i += 2) {
            mx = dev::max3(mx, xc[i], xc[i + 1]);
            const float2 z = dev::fma2(make_float2(xc[i], xc[i + 1]), sc, nm);
            const float2 pp = make_float2(dev::ex2(z.x), dev::ex2(z.y));
            const uint32_t w = dev::pack_bf16x2(pp.x, pp.y);
            pw[(kPer / 2) * r + i / 2] = w;
            e = dev::add2(e, pp);
            q = dev::add2(q, make_float2(dev::bf16_lo(w), dev::bf16_hi(w)));
        }
    }
    if (DUP) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    se = e.x + e.y;
    sr = q.x + q.y;
    return mx * scale_log2;                          // the scale is positive
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_prefix(PrefixArgs a, const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
    using L = PreLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* k_full = bars;                  // [kKSlots] a K slot holds its stage
    uint64_t* k_empty = k_full + L::kKSlots;  // [kKSlots] the Q K^T reading it has completed
    uint64_t* v_full = k_empty + L::kKSlots;  // [kVSlots]
    uint64_t* v_empty = v_full + L::kVSlots;  // [kVSlots] the P V reading it has completed
    uint64_t* q_full = v_empty + L::kVSlots;  // the item's Q tile is written
    uint64_t* q_free = q_full + 1;            // the item's last Q K^T has completed
    uint64_t* s_full = q_free + 1;            // [2] S of a stage is in its buffer
    uint64_t* pv_done = s_full + 2;           // [2] the P V reading P over the buffer has completed
    uint64_t* p_full = pv_done + 2;           // P of a stage is written (over its S)
    uint64_t* p_free = p_full + 1;            // its P V has completed
    uint64_t* o_full = p_free + 1;            // [2] an item's last P V has completed
    uint64_t* o_free = o_full + 2;            // [2] the epilogue has read the item's O
    uint64_t* ml_full = o_free + 2;           // an item's row state is written
    uint64_t* ml_free = ml_full + 1;          // ... and read
    uint64_t* mma_done = ml_free + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 16);
    float* ml = reinterpret_cast<float*>(smem + L::kOffML);

    // the per-request pass, launched after this one, may take the other SMs now
    dev::pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t first_item = blockIdx.x, item_step = gridDim.x;
    const int32_t n_mine = first_item < a.n_items ? (a.n_items - first_item + item_step - 1) / item_step : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < L::kKSlots; ++s) {
            dev::mbar_init(&k_full[s], 1);
            dev::mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < L::kVSlots; ++s) {
            dev::mbar_init(&v_full[s], 1);
            dev::mbar_init(&v_empty[s], 1);
        }
        dev::mbar_init(q_full, 128);
        dev::mbar_init(q_free, 1);
        for (int b = 0; b < 2; ++b) {
            dev::mbar_init(&s_full[b], 1);
            dev::mbar_init(&pv_done[b], 1);
            dev::mbar_init(&o_full[b], 1);
            dev::mbar_init(&o_free[b], 128);
        }
        dev::mbar_init(p_full, 128);
        dev::mbar_init(p_free, 1);
        dev::mbar_init(ml_full, 128);
        dev::mbar_init(ml_free, 128);
        dev::mbar_init(mma_done, 2);
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

    if (warp == 0 || warp == kVWarp) {
        // ------------------------------------------------ TMA producers
        // Stage g of the CTA goes to slot g % slots of its ring.  Block ids
        // are read 32 at a time (four stages), one batch ahead and, for the
        // next item, while the current one streams.
        const bool is_k = warp == 0;
        const CUtensorMap* tm = is_k ? &tmK : &tmV;
        const int nslots = is_k ? L::kKSlots : L::kVSlots;
        uint64_t* full = is_k ? k_full : v_full;
        uint64_t* empty = is_k ? k_empty : v_empty;
        uint8_t* const ring = smem + (is_k ? L::kOffK : L::kOffV);
        if (lane == 0) dev::tma_prefetch_desc(tm);
        constexpr int kStagesPerBatch = 32 / kBlkPerStage;
        ItemCursor ic(a.items, first_item, item_step, n_mine);
        auto fetch = [&](const PrefixItem& it, int32_t batch) -> int32_t {
            const int32_t blk = it.tok0 / kBlockSize + batch * 32 + lane;
            // past the chunk: rows beyond the cache, which TMA fills with zeros
            return blk < it.tok1 / kBlockSize ? __ldg(a.bt + (int64_t)it.bt_row * a.max_blocks + blk) * kBlockSize
                                              : a.num_blocks * kBlockSize;
        };
        uint32_t g = 0;
        bool ok = true;
        int32_t nxt = n_mine > 0 ? fetch(ic.cur, 0) : 0;
        for (; ok && ic.li < n_mine; ic.advance()) {
            const PrefixItem& it = ic.cur;
            const int32_t ns = stages_of(it);
            const int32_t nb = (ns + kStagesPerBatch - 1) / kStagesPerBatch;
            int32_t cur = 0;
            for (int32_t j = 0; ok && j < ns; ++j, ++g) {
                if (j % kStagesPerBatch == 0) {
                    const int32_t batch = j / kStagesPerBatch;
                    cur = nxt;
                    // the next batch of this item, else the first of the next item
                    nxt = batch + 1 < nb ? fetch(it, batch + 1) : (ic.has_next() ? fetch(ic.nxt, 0) : 0);
                }
                // lane i < 8 issues the boxes of the stage's block i
                const int32_t trow = __shfl_sync(0xffffffffu, cur, (j % kStagesPerBatch) * kBlkPerStage + (lane & 7));
                const int s = g % nslots;
                if (lane == 0) {
                    if (g >= (uint32_t)nslots && !dev::mbar_wait(&empty[s], ((g / nslots) - 1) & 1, abort_flag, a.err))
                        ok = false;
                    else
                        dev::mbar_arrive_expect_tx(&full[s], L::kKV);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (lane < kBlkPerStage) {
                    uint8_t* dst = ring + s * L::kKV + lane * (kBlockSize * 128);
#pragma unroll
                    for (int hf = 0; hf < L::kHalves; ++hf)
                        dev::tma_load_3d(dst + hf * (kStage * 128), tm, &full[s], hf * 64, it.head, trow);
                }
            }
        }
        if (lane == 0) {
            // never leave with copies in flight (each slot's latest load only)
            volatile int never = 0;
            for (uint32_t j = g; j > 0 && j + nslots > g; --j)
                dev::mbar_wait(&full[(j - 1) % nslots], ((j - 1) / nslots) & 1, &never, a.err);
        }
        __syncwarp();
    } else if (warp == 1 || warp == kPVWarp) {
        // ------------------------------------------------ MMA issuers
        // Issuing a tcgen05.mma returns about when the tensor core takes it, so
        // one thread that issued both kinds would spend its barrier checks
        // with the tensor core idle: lane 0 of warp 1 issues every Q K^T,
        // lane 0 of warp 3 every P V.  Q K^T(g) overwrites the buffer that held
        // P(g - 2), so it waits for that P V to have completed.
        if (lane == 0) {
            ItemCursor ic(a.items, first_item, item_step, n_mine);
            bool ok = true;
            uint32_t g = 0;
            if (warp == 1) {
                constexpr uint32_t idesc_qk = dev::idesc_bf16_f32(128, kStage, false, false);
                const uint32_t q_base = dev::smem_u32(smem + L::kOffQ);
                const uint32_t k_ring = dev::smem_u32(smem + L::kOffK);
                for (; ok && ic.li < n_mine; ic.advance()) {
                    const int32_t li = ic.li, ns = stages_of(ic.cur);
                    // the item's Q tile is written
                    ok = dev::mbar_wait(q_full, li & 1, abort_flag, a.err);
                    for (int32_t j = 0; ok && j < ns; ++j, ++g) {
                        const uint32_t s = g % L::kKSlots;
                        if (g >= 2 && !dev::mbar_wait(&pv_done[g & 1], ((g >> 1) - 1) & 1, abort_flag, a.err)) {
                            ok = false;
                            break;
                        }
                        if (!dev::mbar_wait(&k_full[s], (g / L::kKSlots) & 1, abort_flag, a.err)) {
                            ok = false;
                            break;
                        }
                        dev::tc_fence_after();
                        const uint32_t k_base = k_ring + s * L::kKV;
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint64_t ad =
                                dev::smem_desc_sw128(q_base + (k >> 2) * (128 * 128) + (k & 3) * 32, 16, 1024);
                            const uint64_t bd =
                                dev::smem_desc_sw128(k_base + (k >> 2) * (kStage * 128) + (k & 3) * 32, 16, 1024);
                            dev::tc_mma_ss(tmem + L::kColS + (g & 1) * 128, ad, bd, idesc_qk, k > 0 ? 1u : 0u);
                        }
                        dev::tc_commit(&s_full[g & 1]);
                        dev::tc_commit(&k_empty[s]);
                        if (j + 1 == ns) dev::tc_commit(q_free);
                    }
                }
            } else {
                constexpr uint32_t idesc_pv = dev::idesc_bf16_f32(128, D, false, true);
                const uint32_t v_ring = dev::smem_u32(smem + L::kOffV);
                for (; ok && ic.li < n_mine; ic.advance()) {
                    const int32_t li = ic.li, ns = stages_of(ic.cur);
                    const int b = li & 1;
                    // the first P V of an item starts its O buffer afresh, once the
                    // epilogue has read what the item two before left there
                    if (li >= 2) ok = dev::mbar_wait(&o_free[b], ((li >> 1) - 1) & 1, abort_flag, a.err);
                    for (int32_t j = 0; ok && j < ns; ++j, ++g) {
                        // O(b) (+)= P(g) V(g), P (bf16 pairs) over S buffer g % 2
                        const uint32_t s = g % L::kVSlots;
                        if (!dev::mbar_wait(p_full, g & 1, abort_flag, a.err) ||
                            !dev::mbar_wait(&v_full[s], (g / L::kVSlots) & 1, abort_flag, a.err)) {
                            ok = false;
                            break;
                        }
                        dev::tc_fence_after();
                        const uint32_t v_base = v_ring + s * L::kKV;
#pragma unroll
                        for (int k = 0; k < kStage / 16; ++k) {
                            const uint64_t bd = dev::smem_desc_sw128(v_base + k * (16 * 128), kStage * 128, 1024);
                            dev::tc_mma_ts(tmem + L::kColO + b * D, tmem + L::kColS + (g & 1) * 128 + k * 8, bd,
                                           idesc_pv, (j == 0 && k == 0) ? 0u : 1u);
                        }
                        dev::tc_commit(p_free);
                        dev::tc_commit(&pv_done[g & 1]);
                        dev::tc_commit(&v_empty[s]);
                        if (j + 1 == ns) dev::tc_commit(&o_full[b]);
                    }
                }
            }
            // every MMA of this thread has retired before tensor memory is freed
            dev::tc_commit(mma_done);
            volatile int never = 0;
            dev::mbar_wait(mma_done, 0, &never, a.err);
        }
        __syncwarp();
    } else if (warp >= kSoftWarp0 && warp < kEpiWarp0) {
        // ------------------------------------------------ softmax
        // Row state: m_ref is the reference the exponentials of new stages use;
        // O and the two row sums are relative to m_used.  When a stage's
        // maximum exceeds m_ref by more than 2^kRescaleLog2 (but not by
        // 2^kRedoLog2), its P is still computed against the old reference
        // (values up to 2^kRedoLog2, well inside bf16 and fp32 range) and the
        // move of O and the sums to the new reference is made at the next
        // stage, once this stage's P V has completed.  A larger jump computes
        // the stage again against the new maximum, with O rescaled before its
        // P V.
        const int quarter = warp & 3;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        bool ok = true;
        uint32_t g = 0;
        ItemCursor ic(a.items, first_item, item_step, n_mine);
        for (; ok && ic.li < n_mine; ic.advance()) {
            const PrefixItem& it = ic.cur;
            const int32_t li = ic.li, ns = stages_of(it), n_tok = it.tok1 - it.tok0;
            const bool dup = dup_of(it);
            const int copy = dup ? (lane >> 4) : 0;
            const int b = li & 1;
            // a warp whose rows are all padding keeps only the barrier protocol
            const bool live = (dup ? quarter * 16 : quarter * 32) < it.nrows;
            const uint32_t o_addr = tmem + lane_base + L::kColO + b * D;
            float m_ref = -INFINITY, m_used = -INFINITY, l_exact = 0.f, l_round = 0.f;
            for (int32_t j = 0; j < ns; ++j, ++g) {
                bool got = dev::mbar_wait(&s_full[g & 1], (g >> 1) & 1, abort_flag, a.err);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                dev::tc_fence_after();
                const uint32_t s_addr = tmem + lane_base + L::kColS + (g & 1) * 128;
                const int32_t n_valid = min(kStage, n_tok - j * kStage);
                const bool mask = n_valid < kStage;          // the chunk's last stage
                float o_scale = 1.f;
                if (m_used != m_ref) {                       // a move owed by the previous stage
                    const float f = dev::ex2(m_used - m_ref);
                    l_exact *= f;
                    l_round *= f;
                    o_scale = f;
                    m_used = m_ref;
                }
                uint32_t pw[kStage / 2];
                if (live) {
                    if (m_ref == -INFINITY) {                // the item's first stage: the row maximum first
                        const float mx = dup ? (mask ? s_rowmax<true, true>(s_addr, copy, n_valid)
                                                     : s_rowmax<true, false>(s_addr, copy, n_valid))
                                             : (mask ? s_rowmax<false, true>(s_addr, copy, n_valid)
                                                     : s_rowmax<false, false>(s_addr, copy, n_valid));
                        m_ref = m_used = mx * a.scale_log2;
                    }
                    float se = 0.f, sr = 0.f;
#pragma unroll 1
                    for (int attempt = 0;; ++attempt) {
                        const float mx =
                            dup ? (mask ? s_exps<true, true>(s_addr, copy, n_valid, a.scale_log2, m_ref, pw, se, sr)
                                        : s_exps<true, false>(s_addr, copy, n_valid, a.scale_log2, m_ref, pw, se, sr))
                                : (mask ? s_exps<false, true>(s_addr, copy, n_valid, a.scale_log2, m_ref, pw, se, sr)
                                        : s_exps<false, false>(s_addr, copy, n_valid, a.scale_log2, m_ref, pw, se, sr));
                        if (attempt == 0 && mx > m_ref + kRedoLog2) {
                            // a jump too large to carry: this stage again, against mx
                            const float f = dev::ex2(m_ref - mx);
                            l_exact *= f;
                            l_round *= f;
                            o_scale *= f;
                            m_ref = m_used = mx;
                            continue;
                        }
                        if (mx > m_ref + kRescaleLog2) m_ref = mx;   // moved at the next stage
                        break;
                    }
                    l_exact += se;
                    l_round += sr;
                }
                // P(g - 1) V has completed: O is up to date
                if (g >= 1) {
                    got = dev::mbar_wait(p_free, (g - 1) & 1, abort_flag, a.err);
                    if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                }
                if (__any_sync(0xffffffffu, o_scale != 1.f)) {
                    dev::tc_fence_after();
                    if (dup) {
                        // lane j's row: threads j and j + 16 take 64 columns each
#pragma unroll 1
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t ov[16];
                            dev::tmem_ld16x2_x16<D / 2>(o_addr + c * 16, ov);
                            dev::tc_wait_ld();
#pragma unroll
                            for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * o_scale);
                            dev::tmem_st16x2_x16<D / 2>(o_addr + c * 16, ov);
                        }
                    } else {
#pragma unroll 1
                        for (int c = 0; c < D / 16; ++c) {
                            uint32_t ov[16];
                            dev::tmem_ld16(o_addr + c * 16, ov);
                            dev::tc_wait_ld();
#pragma unroll
                            for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * o_scale);
                            dev::tmem_st16(o_addr + c * 16, ov);
                        }
                    }
                }
                // P over the S it came from (every thread has read all of its S)
                if (live) {
                    if (dup) {
                        // lane j: threads j and j + 16 write tokens [0, 64) and [64, 128)
                        uint32_t pv[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) pv[i] = pw[i];
                        dev::tmem_st16x2_x32<32>(s_addr, pv);
                    } else {
                        uint32_t p0[32], p1[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            p0[i] = pw[i];
                            p1[i] = pw[32 + i];
                        }
                        dev::tmem_st32(s_addr, p0);
                        dev::tmem_st32(s_addr + 32, p1);
                    }
                }
                dev::tc_wait_st();
                dev::tc_fence_before();
                dev::mbar_arrive(p_full);
            }
            if (!ok) break;
            // the item's row state for the epilogue, once it has read the last one
            if (li >= 1) {
                bool got = dev::mbar_wait(ml_free, (li - 1) & 1, abort_flag, a.err);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            }
            const int t = quarter * 32 + lane;
            ml[t] = m_used;
            ml[128 + t] = l_exact;
            ml[256 + t] = l_round;
            dev::mbar_arrive(ml_full);
        }
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------ Q loader and epilogue
        const int quarter = warp & 3;
        const int t = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        uint8_t* const qtile = smem + L::kOffQ;
        // query row of tile row t of an item: 16-byte pieces, in registers
        uint4 qv[D / 8];
        auto fetch_q = [&](const PrefixItem& it) {
            const int32_t rr = real_row(t, dup_of(it));
            if (rr < it.nrows) {
                const int32_t i = it.row0 + rr;
                const int32_t member = __ldg(a.members + it.moff + i / a.G);
                const uint4* src =
                    reinterpret_cast<const uint4*>(a.q + ((int64_t)member * a.Hq + it.head * a.G + i % a.G) * D);
#pragma unroll
                for (int c = 0; c < D / 8; ++c) qv[c] = __ldg(src + c);
            } else {
#pragma unroll
                for (int c = 0; c < D / 8; ++c) qv[c] = make_uint4(0, 0, 0, 0);
            }
        };
        auto store_q = [&]() {
#pragma unroll
            for (int c = 0; c < D / 8; ++c)
                *reinterpret_cast<uint4*>(qtile + sw128_off(t, c >> 3, c & 7, 128 * 128)) = qv[c];
            dev::fence_proxy_async_smem();
            dev::mbar_arrive(q_full);
        };
        // Staging: this warp's 32 slots of 128 bytes, 16-byte chunks swizzled by
        // slot, so that both the slot-per-thread writes and the line-per-eight-
        // threads reads are free of bank conflicts.
        uint8_t* const stg_w = smem + L::kOffStg + quarter * (32 * 128);
        bool ok = true;
        ItemCursor ic(a.items, first_item, item_step, n_mine);
        if (n_mine > 0) {
            fetch_q(ic.cur);
            store_q();
        }
        if (ic.has_next()) fetch_q(ic.nxt);
        int32_t stg_i = 0;                                // staging buffer toggle
        for (; ok && ic.li < n_mine; ic.advance()) {
            const PrefixItem it = ic.cur;
            const int32_t li = ic.li;
            if (ic.has_next()) {
                // the Q tile is free once the item's last Q K^T has completed
                bool got = dev::mbar_wait(q_free, li & 1, abort_flag, a.err);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                store_q();
                if (li + 2 < n_mine) fetch_q(load_item(a.items, first_item + (li + 2) * item_step));
            }
            // epilogue of item li: normalise the rows and write the partials
            const int b = li & 1;
            const bool dup = dup_of(it);
            {
                bool got = dev::mbar_wait(ml_full, li & 1, abort_flag, a.err);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            }
            const float m_row = ml[t];
            float l_exact = ml[128 + t], l_round = ml[256 + t];
            dev::mbar_arrive(ml_free);
            {
                bool got = dev::mbar_wait(&o_full[b], (li >> 1) & 1, abort_flag, a.err);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            }
            dev::tc_fence_after();
            const bool live = (dup ? quarter * 16 : quarter * 32) < it.nrows;
            if (live) {
                // the two halves of a duplicated row share m; their sums add up
                if (dup) {
                    l_exact += __shfl_xor_sync(0xffffffffu, l_exact, 16);
                    l_round += __shfl_xor_sync(0xffffffffu, l_round, 16);
                }
                const float inv = 1.f / l_round;
                const int32_t rr = real_row(t, dup);
                const int copy = dup ? (lane >> 4) : 0;
                if (rr < it.nrows && copy == 0)
                    a.part_lse[it.part_row0 + rr] = (m_row + __log2f(l_exact)) * 0.69314718055994531f;
                // 32-column passes: thread (slot) l holds 32 floats of one row
                // (rows of this warp's quarter; a duplicated row's two halves go
                // to threads j and j + 16)
                const int npass = dup ? D / 64 : D / 32;
                const int rows_here = min(dup ? 16 : 32, it.nrows - (dup ? quarter * 16 : quarter * 32));
#pragma unroll 1
                for (int ps = 0; ps < npass; ++ps) {
                    uint32_t ov[32];
                    if (dup)
                        dev::tmem_ld16x2_x32<D / 2>(tmem + lane_base + L::kColO + b * D + ps * 32, ov);
                    else
                        dev::tmem_ld32(tmem + lane_base + L::kColO + b * D + ps * 32, ov);
                    dev::tc_wait_ld();
                    uint8_t* stg = stg_w + stg_i * L::kStageBytes;
                    stg_i ^= 1;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<float4*>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                            make_float4(__uint_as_float(ov[4 * c]) * inv, __uint_as_float(ov[4 * c + 1]) * inv,
                                        __uint_as_float(ov[4 * c + 2]) * inv, __uint_as_float(ov[4 * c + 3]) * inv);
                    __syncwarp();
                    // eight threads per slot: slot sl's 128 bytes go to one line of
                    // its row's partial
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int sl = 4 * k + (lane >> 3), c = lane & 7;
                        const int row_in = dup ? (sl & 15) : sl;           // row within this warp's rows
                        const int col = dup ? (sl >> 4) * (D / 2) + ps * 32 : ps * 32;
                        if (row_in < rows_here) {
                            const float4 v = *reinterpret_cast<const float4*>(stg + sl * 128 + ((c ^ (sl & 7)) << 4));
                            const int32_t row = (dup ? quarter * 16 : quarter * 32) + row_in;
                            *reinterpret_cast<float4*>(a.part_o + ((int64_t)it.part_row0 + row) * D + col + c * 4) = v;
                        }
                    }
                }
            }
            dev::tc_fence_before();
            dev::mbar_arrive(&o_free[b]);
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
    cudaError_t e = cudaFuncSetAttribute(k_prefix<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (max_ctas > 0) sms = std::min(sms, max_ctas);
    const int grid = std::max(1, std::min(sms, a.n_items));
    k_prefix<D><<<grid, kThreads, L::kAlloc, stream>>>(a, tk, tv);
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
