// Internal declarations shared by the host and device parts of libfca_b200.
//
// Work-list records and the plan object.  Nothing here is part of the C ABI
// (include/fca.h); the layout of these records may change between builds.
#pragma once

#include <cstdint>
#include <vector>
#include <cuda.h>
#include <cuda_runtime.h>

#include "fca.h"

namespace fca {

constexpr int kBlockSize = 16;        // tokens per paged block (the only size built)
constexpr int kPrefixTileRows = 128;  // stacked query rows per tcgen05 tile (MMA M)
constexpr int kStageTokens = 128;     // tokens per pipeline stage of the grouped pass
constexpr int kMaxGqa = 16;           // query heads per KV head handled by the own pass
constexpr int kMaxRequests = 16384;   // groups are sorted in one CTA's shared memory
constexpr int kMaxRequestsFallback = 4096;  // all-pairs LCP path (see fca_plan.cu)

// Device error word bits (fca_check_device_status).
constexpr int32_t kErrWaitTimeout = 1;     // a bounded mbarrier wait ran out
constexpr int32_t kErrBadItem = 2;         // a work item failed its own range check
constexpr int32_t kErrPlanInternal = 4;    // a planner consistency check failed (no write done)
constexpr int32_t kErrUpdateRefused = 32;  // an asynchronous fca_plan_update was refused (plan unchanged)

// Raised by the work-list kernel of fca_paged_decode_static, which cannot
// return an error to the host: the request is skipped (out 0, lse -inf).
constexpr int32_t kErrStaticSeqLen = 8;    // seq_len outside [1, max_blocks * block_size]
constexpr int32_t kErrStaticBlockId = 16;  // a used table entry outside [0, num_blocks)

// Size of the fixed device array behind fca_paged_decode_static.
constexpr size_t kStaticScratchBytes = size_t(64) << 20;

// Per-SM throughput of the two passes when they run side by side, measured on
// B200 (K/V bytes a second per SM): the grouped pass streams a group's tokens
// once per 128-row query tile, the per-request pass its own tokens.  Used to
// choose how many SMs the grouped pass starts on and to size its chunks.
constexpr double kPrefixGBsPerSM = 18.0;
constexpr double kSuffixGBsPerSM = 49.0;

// Default of fca_plan_opts.min_saved_blocks: a group is used only if sharing
// it saves at least this many block reads, (members - 1) x its length in
// blocks.  A grouped-pass work item costs about as much as streaming 32 blocks
// of one KV head in the per-request pass (item set-up, query-tile load and
// epilogue), so smaller groups make the step slower: on 512 pairs of requests
// sharing 1-16 blocks, keeping every group took 745 us a step against 522 for
// the flat decode.
constexpr int32_t kDefaultMinSavedBlocks = 32;

// Group partials per request whose rows the planner records for the merge
// (more take the chain walk).
constexpr int kMergeRec = 8;

// Shortest chunk the per-request pass splits a request's own tokens into.
// Longer chunks mean fewer partial rows to write and merge; a sweep of 256,
// 384 and 512 on the four large workloads favoured 512 (forest 204 -> 195 us
// a step, the others unchanged); with the per-request pass taking over the
// grouped pass's SMs, 384, 768 and 1024 were within 1% of 512 on all four.
constexpr int32_t kMinOwnChunk = 512;

// Planner status bits (read back inside fca_plan).
constexpr int32_t kPlanBadSeqLen = 1;
constexpr int32_t kPlanBadBlockId = 2;
constexpr int32_t kPlanInconsistent = 4;   // block ids do not identify prefixes
constexpr int32_t kPlanTooManyGroups = 8;
constexpr int32_t kPlanUpdateMismatch = 16;   // fca_plan_update: a shared entry or length no longer fits

// One tile of the grouped prefix pass: rows [row0, row0 + nrows) of a
// group's stacked queries (member i / G, query head head * G + i % G; the
// group's members start at members[moff]), against tokens [tok0, tok1) of the
// table row of request `bt_row`.
struct PrefixItem {
    int32_t moff, head, row0, nrows;
    int32_t tok0, tok1, bt_row, part_row0;   // partial row of stacked row row0
};

// One chunk of a request's own pass: the G query heads of KV head `head`
// against tokens [tok0, tok1) of request `request`'s table.
struct SuffixItem {
    int32_t request, head, tok0, tok1;
    int32_t part_row0, pad0, pad1, pad2;     // first of G partial rows
};

// Sizes the planner computes on the device and fca_plan reads back once.
struct PlanHeader {
    int32_t status;
    int32_t n_groups;
    int32_t n_member_entries;   // sum of group sizes
    int32_t max_depth;
    int32_t split_tokens;       // chunk target of the per-request pass
    int32_t prefix_split_tokens;// chunk target of the grouped pass
    int32_t n_prefix_items;
    int32_t n_suffix_items;
    int32_t n_prefix_partials;  // partial rows written by the grouped pass
    int32_t n_suffix_partials;
    int32_t n_chain_entries;    // sum over requests of their group depth
    int64_t unique_kv_tokens;
    int64_t fca_kv_tokens;      // token-blocks the FCA passes read (per KV head)
    int64_t flat_kv_tokens;
    int64_t prefix_tok_sum;     // sum over groups of their token count
    int64_t suffix_tok_sum;
    int64_t prefix_tile_tok_sum;// sum over groups of token count x 128-row query tiles
    int64_t own_chunk_cap;      // own-pass chunks any update can need (plans with asynchronous updates)
};

// Remember e (if it is an error) as the calling thread's last CUDA error.
cudaError_t note_cuda(cudaError_t e);

// TMA descriptor of a K or V cache [num_blocks * 16][Hkv][D] bf16 (fca_api.cu).
bool make_cache_map(CUtensorMap* map, const void* base, int32_t num_blocks, int32_t Hkv, int32_t D);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace fca

// The plan object behind fca_plan_t.
struct fca_plan_s {
    int device = 0;
    int32_t R = 0, max_blocks = 0, block_size = 0, num_blocks = 0;
    int32_t Hq = 0, Hkv = 0, D = 0, G = 0;
    fca_plan_opts opts{};
    bool flat = false;
    fca::PlanHeader hdr{};
    size_t workspace_bytes = 0;
    int64_t cap_suffix_items = 0;    // capacity of suffix_items (fca_plan_update may need more)
    int64_t cap_partials = 0;        // capacity of part_o / part_lse, in rows
    bool async_update = false;       // FCA_PLAN_ASYNC_UPDATE: updates stay on the device; the
                                     // per-request pass reads its item count from sched[2]
    void* upd_scratch = nullptr;     // temporaries of asynchronous updates

    // copies of the inputs
    int32_t* bt = nullptr;           // [R][max_blocks]
    int32_t* seq_lens = nullptr;     // [R]
    // forest, canonical order
    int32_t* g_a = nullptr;          // [n_groups]
    int32_t* g_b = nullptr;
    int32_t* g_parent = nullptr;
    int32_t* g_moff = nullptr;
    int32_t* g_nm = nullptr;
    int32_t* g_nch = nullptr;        // split chunks of the group's token range
    int32_t* g_chunk = nullptr;      // tokens per chunk (last one may be shorter)
    int32_t* g_part = nullptr;       // partial row of (group, head 0, chunk 0, row 0)
    int32_t* g_wa = nullptr;         // first block of the group's grouped-pass items (its a, or
                                     // its parent's when the parent is folded into its children)
    int32_t* members = nullptr;      // [n_member_entries]
    int32_t* suffix_start = nullptr; // [R] blocks
    int32_t* chain_off = nullptr;    // [R + 1] into chain_g / chain_pos
    int32_t* chain_g = nullptr;      // groups of request r, root first
    int32_t* chain_pos = nullptr;    // r's index among the group's members
    int32_t* s_nch = nullptr;        // [R] chunks of r's own pass
    int32_t* s_chunk = nullptr;      // [R] tokens per chunk (last one may be shorter)
    int32_t* sched = nullptr;        // [4] work counters of the two passes (self-resetting)
    int32_t* s_part = nullptr;       // [R] partial row of (r, head 0, chunk 0)
    fca::PrefixItem* prefix_items = nullptr;
    fca::SuffixItem* suffix_items = nullptr;
    float* part_o = nullptr;         // [n_partials][D]
    float* part_lse = nullptr;       // [n_partials]
    int32_t* dev_status = nullptr;   // device error word
    int32_t* m_ng = nullptr;         // [R] partials per KV head from r's groups
    int2* m_rec = nullptr;           // [R][kMergeRec] where they are: row of (KV head h, query head i)
                                     // = x + h y + i (chain order; unused when m_ng > kMergeRec)

    // every cudaMalloc the plan owns (freed by fca_plan_destroy)
    std::vector<void*> dev_allocs;
};
