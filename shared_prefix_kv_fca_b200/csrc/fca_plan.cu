// Group discovery and work-list construction for Forest Cascade Attention.
//
// "ZoRRo Inference & Forest Cascade Attention", "Core Mechanism" step 1:
// discover the groups of requests that share a KV-cache prefix.  Sharing is
// by physical block: requests that start with the same prompt reference the
// same physical blocks ("PagedAttention vs. RadixAttention", "How
// PagedAttention Works", step 4), and only full blocks are shareable (a block
// that is still being written is copied before it diverges).
//
// The forest is the trie of the requests' full-block id sequences: a node is
// a prefix, its member set is the requests whose tables start with it, and a
// group is a maximal run of depths over which the member set does not change
// (and has at least min_group_size members).  A group shorter than
// min_shared_blocks, or one whose sharing saves fewer than min_saved_blocks
// block reads ((members - 1) x length), is folded: its interval passes to the
// groups below it, or to its members' own passes.
//
// Fast path (every table produced by a prefix-caching allocator).  A trie node
// at depth k + 1 is identified by the physical block at logical index k,
// because a cached block's identity already stands for its whole prefix
// ("How vLLM Implements Prefix Caching": each block's hash chains its parent's
// hash, so equal blocks imply equal prefixes).  The planner checks that
// property on the device -- every block id appears at one logical index only,
// and all requests holding block b at index k hold the same block at k - 1 --
// which makes "same block at index k" equivalent to "same prefix of length
// k + 1".  Then a node's member count and smallest member are per-block
// atomics, and each request's groups are the runs of constant count along its
// row.
//
// Fallback (tables that break the property).  Each request computes its
// longest common full-block prefix with every other request, sorts those
// lengths, and reads a node's count and smallest member off the sorted list.
// Exact for any input; O(R^2) work, used only when the check fails and
// R <= kMaxRequestsFallback.
//
// Canonical order of the output: groups by (first block, smallest member);
// members ascending.  One CTA sorts the groups in shared memory.
#include <algorithm>
#include <mutex>
#include <cstdio>
#include <cstring>
#include <vector>

#include "fca_internal.h"

// A group's grouped-pass work up to this many times the chunk target stays one
// item (sweep of 1.0 / 1.5 / 2.0 on four workloads: 1.5 and 2.0 took the
// llama8b step from 141 to 139 us and the forest's from 201 to 193 once its
// root is folded into its prompts' items; 1.0 is the plain ceiling).
constexpr double kWholeItem = 1.5;

namespace fca {
namespace {


struct RawGroup {
    int32_t a, b, owner, nm;
    int32_t parent_a, parent_owner, pad0, pad1;
};

struct PlanScratch {
    int32_t* nfull;        // [R]
    int32_t* owner;        // [NB]
    int32_t* count;        // [NB]
    int32_t* pos;          // [NB]
    int32_t* valid;        // [NB] valid tokens per block (for unique bytes)
    int32_t* n_emit;       // [R]
    int32_t* row_goff;     // [R + 1]
    int32_t* fill;         // [R]
    int32_t* n_raw;        // [1]
    RawGroup* raw;         // [R]
    uint64_t* keys;        // [R] canonical (a << 32 | owner)
    int32_t* g_item_off;   // [R + 1]
    int32_t* s_item_off;   // [R + 1]
    int32_t* gwork;        // [4 R] per group: children's members, tiles, count, non-leaf count
    PlanHeader* hdr;       // [1]
};

__device__ __forceinline__ int32_t ceil_div_dev(int32_t a, int32_t b) { return (a + b - 1) / b; }

// Own-pass items are ordered by length (in blocks, capped) so that the
// longest are taken first.
constexpr int32_t kBins = 1024;
__device__ __forceinline__ int32_t length_bin(int32_t tokens) {
    return min(kBins - 1, (tokens + kBlockSize - 1) / kBlockSize);
}

// ------------------------------------------------------------ validation

// Thread (r, j): checks seq_lens[r] (j == 0) and table entry j if it is read.
__global__ void k_validate(const int32_t* __restrict__ bt, int32_t MB, const int32_t* __restrict__ sl,
                           int32_t R, int32_t NB, int32_t* __restrict__ nfull, int32_t* __restrict__ valid,
                           PlanHeader* hdr) {
    const int64_t total = (int64_t)R * MB;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t r = (int32_t)(i / MB), j = (int32_t)(i % MB);
        const int32_t L = sl[r];
        const bool len_ok = L >= 1 && (int64_t)L <= (int64_t)MB * kBlockSize;
        if (j == 0) {
            nfull[r] = len_ok ? L / kBlockSize : 0;
            if (!len_ok) atomicOr(&hdr->status, kPlanBadSeqLen);
        }
        if (!len_ok || j >= ceil_div_dev(L, kBlockSize)) continue;
        const int32_t b = bt[i];
        if (b < 0 || b >= NB) {
            atomicOr(&hdr->status, kPlanBadBlockId);
            continue;
        }
        atomicMax(&valid[b], min(kBlockSize, L - j * kBlockSize));
    }
}

// Sum of valid tokens over all blocks (each physical block once).
__global__ void k_unique_tokens(const int32_t* __restrict__ valid, int32_t NB, PlanHeader* hdr) {
    int64_t acc = 0;
    for (int32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < NB; i += gridDim.x * blockDim.x) acc += valid[i];
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0 && acc) atomicAdd(reinterpret_cast<unsigned long long*>(&hdr->unique_kv_tokens),
                                                  (unsigned long long)acc);
}

// ------------------------------------------------------------ fast path

__global__ void k_block_keys(const int32_t* __restrict__ bt, int32_t MB, int32_t R,
                             const int32_t* __restrict__ nfull, int32_t* __restrict__ owner,
                             int32_t* __restrict__ count, int32_t* __restrict__ pos, PlanHeader* hdr) {
    if (hdr->status & (kPlanBadSeqLen | kPlanBadBlockId)) return;
    const int64_t total = (int64_t)R * MB;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t r = (int32_t)(i / MB), k = (int32_t)(i % MB);
        if (k >= nfull[r]) continue;
        const int32_t b = bt[i];
        atomicMin(&owner[b], r);
        atomicAdd(&count[b], 1);
        const int32_t old = atomicCAS(&pos[b], -1, k);
        if (old != -1 && old != k) atomicOr(&hdr->status, kPlanInconsistent);
    }
}

__global__ void k_check_chain(const int32_t* __restrict__ bt, int32_t MB, int32_t R,
                              const int32_t* __restrict__ nfull, const int32_t* __restrict__ owner,
                              PlanHeader* hdr) {
    if (hdr->status & (kPlanBadSeqLen | kPlanBadBlockId | kPlanInconsistent)) return;
    const int64_t total = (int64_t)R * MB;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t r = (int32_t)(i / MB), k = (int32_t)(i % MB);
        if (k == 0 || k >= nfull[r]) continue;
        const int32_t o = owner[bt[i]];
        if (bt[(int64_t)o * MB + k - 1] != bt[i - 1]) atomicOr(&hdr->status, kPlanInconsistent);
    }
}

// ------------------------------------------------------------ row runs

struct RowArgs {
    const int32_t* bt;
    int32_t MB, R, G, min_group_size, min_shared_blocks, min_saved_blocks, pass;
    const int32_t* nfull;
    const int32_t* owner;
    const int32_t* count;
    PlanScratch s;
    int32_t* suffix_start;
    // pass 1 outputs
    const uint64_t* keys;   // canonical keys (a << 32 | owner), n_groups of them
    const int32_t* g_moff;
    int32_t* members;
    int32_t* chain_g;
    int32_t* err;           // the plan's device error word
};

// Node information for (row, depth index k): member count and smallest member.
struct NodeReader {
    // fast path
    const int32_t* row;
    const int32_t* owner;
    const int32_t* count;
    // fallback: LCPs with all other requests, sorted by (lcp desc, request asc),
    // and the running minimum of the request ids in that order
    const int32_t* sorted_lcp;
    const int32_t* prefix_min;
    int32_t n_others, self;
    bool fallback;

    __device__ void at(int32_t k, int32_t& cnt, int32_t& own) const {
        if (!fallback) {
            const int32_t b = row[k];
            cnt = count[b];
            own = owner[b];
            return;
        }
        // number of others whose LCP with this row exceeds k
        int32_t lo = 0, hi = n_others;
        while (lo < hi) {
            const int32_t mid = (lo + hi) >> 1;
            if (sorted_lcp[mid] > k) lo = mid + 1; else hi = mid;
        }
        cnt = 1 + lo;
        own = lo > 0 ? min(self, prefix_min[lo - 1]) : self;
    }
};

__device__ int32_t find_group(const uint64_t* keys, int32_t n, uint64_t key) {
    int32_t lo = 0, hi = n;
    while (lo < hi) {
        const int32_t mid = (lo + hi) >> 1;
        if (keys[mid] < key) lo = mid + 1; else hi = mid;
    }
    return lo;
}

// One CTA per request.  Pass 0: count the request's groups, set its suffix
// start, and (if it is a group's smallest member) record the group.  Pass 1:
// scatter the request into its groups' member lists and its chain.
__global__ void __launch_bounds__(256) k_row_runs(RowArgs args) {
    extern __shared__ int32_t sm_rows[];
    PlanHeader* hdr = args.s.hdr;
    const int32_t status = hdr->status;
    if (status & (kPlanBadSeqLen | kPlanBadBlockId)) return;
    const bool fallback = (status & kPlanInconsistent) != 0;
    if (fallback && args.R > kMaxRequestsFallback) return;
    const int32_t R = args.R, MB = args.MB;
    const int32_t n_groups = args.pass ? hdr->n_groups : 0;

    for (int32_t r = blockIdx.x; r < R; r += gridDim.x) {
        const int32_t nf = args.nfull[r];
        const int32_t* row = args.bt + (int64_t)r * MB;
        NodeReader nr;
        nr.row = row;
        nr.owner = args.owner;
        nr.count = args.count;
        nr.fallback = fallback;
        nr.self = r;
        nr.n_others = R - 1;
        if (fallback) {
            // LCP with every other request, warp-cooperative compares
            int32_t N = 1;
            while (N < R) N <<= 1;
            uint64_t* key = reinterpret_cast<uint64_t*>(sm_rows);
            const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
            for (int32_t s = warp; s < N; s += nw) {
                if (s >= R || s == r) {
                    if (lane == 0) key[s] = ~0ull;
                    continue;
                }
                const int32_t n = min(nf, args.nfull[s]);
                const int32_t* other = args.bt + (int64_t)s * MB;
                int32_t lcp = n;
                for (int32_t base = 0; base < n; base += 32) {
                    const int32_t k = base + lane;
                    const bool diff = k < n && row[k] != other[k];
                    const uint32_t m = __ballot_sync(0xffffffffu, diff);
                    if (m) {
                        lcp = base + __ffs(m) - 1;
                        break;
                    }
                }
                // ascending key order = lcp descending, then request ascending
                if (lane == 0) key[s] = ((uint64_t)(uint32_t)(0x7FFFFFFF - lcp) << 32) | (uint32_t)s;
            }
            __syncthreads();
            for (int32_t k = 2; k <= N; k <<= 1)
                for (int32_t j = k >> 1; j > 0; j >>= 1) {
                    for (int32_t i = threadIdx.x; i < N; i += blockDim.x) {
                        const int32_t p = i ^ j;
                        if (p > i) {
                            const bool up = (i & k) == 0;
                            const uint64_t x = key[i], y = key[p];
                            if ((x > y) == up) { key[i] = y; key[p] = x; }
                        }
                    }
                    __syncthreads();
                }
            int32_t* lcp_sorted = sm_rows + 2 * N;
            int32_t* pmin = lcp_sorted + N;
            if (threadIdx.x == 0) {
                int32_t m = 0x7FFFFFFF;
                for (int32_t i = 0; i < R - 1; ++i) {
                    lcp_sorted[i] = 0x7FFFFFFF - (int32_t)(key[i] >> 32);
                    m = min(m, (int32_t)(key[i] & 0xFFFFFFFFu));
                    pmin[i] = m;
                }
            }
            __syncthreads();
            nr.sorted_lcp = lcp_sorted;
            nr.prefix_min = pmin;
        }

        // The run scan is short and sequential in the number of runs; one
        // thread walks the change points, the rest of the warp finds them.
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            int32_t cur_start = 0, cur_cnt = 0, cur_own = 0;
            int32_t pending = -1, last_a = -1, last_owner = -1, last_b = 0, n_emit = 0;
            bool done = nf == 0;
            if (!done) {
                nr.at(0, cur_cnt, cur_own);
                if (cur_cnt < args.min_group_size) done = true;
            }
            for (int32_t base = 0; !done && base < nf; base += 32) {
                const int32_t k = base + 1 + lane;     // candidate run end
                int32_t c = 0, o = 0;
                bool is_end = false;
                if (k <= nf) {
                    if (k == nf) {
                        is_end = true;
                    } else {
                        nr.at(k, c, o);
                        int32_t cp, op;
                        nr.at(k - 1, cp, op);
                        is_end = c != cp;
                    }
                }
                uint32_t ends = __ballot_sync(0xffffffffu, is_end);
                while (ends) {
                    const int src = __ffs(ends) - 1;
                    ends &= ends - 1;
                    const int32_t kend = base + 1 + src;
                    const int32_t next_c = __shfl_sync(0xffffffffu, c, src);
                    const int32_t next_o = __shfl_sync(0xffffffffu, o, src);
                    // close the run [cur_start, kend) with count cur_cnt
                    const int32_t eff_a = pending >= 0 ? pending : cur_start;
                    // too short, or saving too few block reads ((members - 1) x length)
                    // to pay for its own work items: fold it
                    if (kend - eff_a < args.min_shared_blocks ||
                        (int64_t)(cur_cnt - 1) * (kend - eff_a) < (int64_t)args.min_saved_blocks) {
                        pending = eff_a;
                    } else {
                        if (args.pass == 0) {
                            if (lane == 0 && cur_own == r) {
                                const int32_t slot = atomicAdd(args.s.n_raw, 1);
                                if (slot < R) {
                                    RawGroup g;
                                    g.a = eff_a;
                                    g.b = kend;
                                    g.owner = r;
                                    g.nm = cur_cnt;
                                    g.parent_a = last_a;
                                    g.parent_owner = last_owner;
                                    g.pad0 = g.pad1 = 0;
                                    args.s.raw[slot] = g;
                                } else {
                                    atomicOr(&hdr->status, kPlanTooManyGroups);
                                }
                            }
                        } else if (lane == 0) {
                            const uint64_t key = ((uint64_t)(uint32_t)eff_a << 32) | (uint32_t)cur_own;
                            const int32_t g = find_group(args.keys, n_groups, key);
                            const int32_t slot = (g < n_groups && args.keys[g] == key) ? atomicAdd(&args.s.fill[g], 1)
                                                                                     : -1;
                            const int32_t c = args.s.row_goff[r] + n_emit;
                            if (slot < 0 || slot >= args.g_moff[g + 1] - args.g_moff[g] || c >= args.s.row_goff[r + 1]) {
                                atomicOr(args.err, kErrPlanInternal);   // never expected; skip the write
                            } else {
                                args.members[args.g_moff[g] + slot] = r;
                                args.chain_g[c] = g;
                            }
                        }
                        pending = -1;
                        last_a = eff_a;
                        last_owner = cur_own;
                        last_b = kend;
                        ++n_emit;
                    }
                    if (kend >= nf || next_c < args.min_group_size) {
                        done = true;
                        break;
                    }
                    cur_start = kend;
                    cur_cnt = next_c;
                    cur_own = next_o;
                }
            }
            if (lane == 0 && args.pass == 0) {
                args.s.n_emit[r] = n_emit;
                args.suffix_start[r] = last_b;
            }
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------ finalize

__device__ int64_t block_sum64(int64_t v, int64_t* red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int64_t t = 0;
    if (threadIdx.x < 32) {
        t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0;
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (threadIdx.x == 0) red[32] = t;
    }
    __syncthreads();
    return red[32];
}

__device__ int32_t block_max32(int32_t v, int64_t* red) {
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (threadIdx.x < 32) {
        int32_t t = threadIdx.x < (blockDim.x >> 5) ? (int32_t)red[threadIdx.x] : 0;
        for (int o = 16; o > 0; o >>= 1) t = max(t, __shfl_xor_sync(0xffffffffu, t, o));
        if (threadIdx.x == 0) red[32] = t;
    }
    __syncthreads();
    return (int32_t)red[32];
}

// Exclusive scan of f(i), i in [0, n), into out[0..n] (out[n] = total).
// Each thread owns a contiguous run; one block-wide pass over the run sums.
template <typename F>
__device__ int64_t block_exclusive_scan(int32_t n, F f, int32_t* out, int64_t* red) {
    const int32_t T = blockDim.x;
    const int32_t per = (n + T - 1) / T;
    const int32_t lo = min(n, (int32_t)threadIdx.x * per), hi = min(n, lo + per);
    int64_t local = 0;
    for (int32_t i = lo; i < hi; ++i) local += f(i);
    // inclusive scan of per-thread sums through shared memory
    __syncthreads();
    red[64 + threadIdx.x] = local;
    __syncthreads();
    for (int32_t off = 1; off < T; off <<= 1) {
        const int64_t v = threadIdx.x >= off ? red[64 + threadIdx.x - off] : 0;
        __syncthreads();
        red[64 + threadIdx.x] += v;
        __syncthreads();
    }
    int64_t run = red[64 + threadIdx.x] - local;
    const int64_t total = red[64 + T - 1];
    for (int32_t i = lo; i < hi; ++i) {
        out[i] = (int32_t)run;
        run += f(i);
    }
    if (threadIdx.x == 0) out[n] = (int32_t)total;
    __syncthreads();
    return total;
}

struct FinalizeArgs {
    PlanScratch s;
    int32_t R, G, Hkv, split_opt, flat;
    const int32_t* seq_lens;
    const int32_t* suffix_start;
    // outputs (canonical order)
    int32_t* g_a;
    int32_t* g_b;
    int32_t* g_parent;
    int32_t* g_nm;
    int32_t* g_moff;     // [R + 1]
    int32_t* g_nch;
    int32_t* g_part;
    int32_t* s_nch;
    int32_t* s_part;
    int32_t* chain_off;  // [R + 1]
    int32_t* g_chunk;
    int32_t* s_chunk;
    int32_t* g_wa;       // first block of each group's grouped-pass items
    int32_t* bin_cursor; // [kBins] first item slot of each length bin, longest first
    int32_t num_sms;
};

// One CTA of 1024 threads.  Shared memory: sort keys (next pow2 of R, 8 B)
// plus 64 + 1024 int64 of reduction space.
__global__ void __launch_bounds__(1024) k_finalize(FinalizeArgs A) {
    extern __shared__ uint64_t sm_fin[];
    PlanHeader* hdr = A.s.hdr;
    if (hdr->status & (kPlanBadSeqLen | kPlanBadBlockId | kPlanTooManyGroups)) return;
    if ((hdr->status & kPlanInconsistent) && A.R > kMaxRequestsFallback) return;
    const int32_t R = A.R, G = A.G;
    const int32_t n = A.flat ? 0 : min(*A.s.n_raw, R);
    int32_t N = 1;
    while (N < n) N <<= 1;
    uint64_t* key = sm_fin;
    int64_t* red = reinterpret_cast<int64_t*>(sm_fin + N);

    for (int32_t i = threadIdx.x; i < N; i += blockDim.x) {
        if (i < n) {
            const RawGroup g = A.s.raw[i];
            key[i] = ((uint64_t)(uint32_t)g.a << 40) | ((uint64_t)(uint32_t)g.owner << 20) | (uint32_t)i;
        } else {
            key[i] = ~0ull;
        }
    }
    __syncthreads();
    for (int32_t k = 2; k <= N; k <<= 1)
        for (int32_t j = k >> 1; j > 0; j >>= 1) {
            for (int32_t i = threadIdx.x; i < N; i += blockDim.x) {
                const int32_t p = i ^ j;
                if (p > i) {
                    const bool up = (i & k) == 0;
                    const uint64_t x = key[i], y = key[p];
                    if ((x > y) == up) { key[i] = y; key[p] = x; }
                }
            }
            __syncthreads();
        }
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) {
        const RawGroup g = A.s.raw[key[i] & 0xFFFFF];
        A.g_a[i] = g.a;
        A.g_b[i] = g.b;
        A.g_nm[i] = g.nm;
        A.s.keys[i] = ((uint64_t)(uint32_t)g.a << 32) | (uint32_t)g.owner;
    }
    __syncthreads();
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) {
        const RawGroup g = A.s.raw[key[i] & 0xFFFFF];
        int32_t par = -1;
        if (g.parent_a >= 0) {
            const uint64_t pk = ((uint64_t)(uint32_t)g.parent_a << 32) | (uint32_t)g.parent_owner;
            par = find_group(A.s.keys, n, pk);
        }
        A.g_parent[i] = par;
    }
    __syncthreads();

    // A group whose members all belong to its child groups, whose children are
    // leaves, and whose children need no more 128-row query tiles than it
    // does, has no work items of its own: each child's items start at the
    // parent's first block instead (a member's tables agree on the parent's
    // interval and the child's), so the parent's blocks are streamed the same
    // number of times, by fewer and longer items, with one partial row per
    // member fewer to write and merge.  (The forest of a system prompt over
    // several prompts: the root's tiles are the prompts' tiles.)
    const int32_t tile_rows = kPrefixTileRows;
    auto tiles_of = [&](int32_t i) { return (A.g_nm[i] * G + tile_rows - 1) / tile_rows; };
    int32_t* c_nm = A.s.gwork;
    int32_t* c_tiles = c_nm + R;
    int32_t* c_count = c_tiles + R;
    int32_t* c_inner = c_count + R;   // children that have children; -1 marks a folded-in parent
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) c_nm[i] = c_tiles[i] = c_count[i] = c_inner[i] = 0;
    __syncthreads();
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) {
        const int32_t par = A.g_parent[i];
        if (par >= 0) {
            atomicAdd(&c_nm[par], A.g_nm[i]);
            atomicAdd(&c_tiles[par], tiles_of(i));
            atomicAdd(&c_count[par], 1);
        }
    }
    __syncthreads();
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) {
        const int32_t par = A.g_parent[i];
        if (par >= 0 && c_count[i] > 0) atomicAdd(&c_inner[par], 1);
    }
    __syncthreads();
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x)
        if (c_count[i] > 0 && c_inner[i] == 0 && c_nm[i] == A.g_nm[i] && c_tiles[i] <= tiles_of(i)) c_inner[i] = -1;
    __syncthreads();
    auto folded_in = [&](int32_t i) { return c_inner[i] < 0; };
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) {
        const int32_t par = A.g_parent[i];
        A.g_wa[i] = (par >= 0 && folded_in(par)) ? A.g_a[par] : A.g_a[i];
    }
    __syncthreads();

    // Chunk targets.  The grouped pass runs one CTA per SM, so aim at about
    // three items per SM; the per-request pass runs one item per warp, eight
    // warps per SM, so aim at about four items per warp, with chunks of at
    // least kMinOwnChunk tokens.  Each group / request then splits its tokens
    // evenly into chunks of at most the target.
    int64_t wp = 0, ws = 0;
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) {
        const int64_t tok = folded_in(i) ? 0 : (int64_t)(A.g_b[i] - A.g_wa[i]) * kBlockSize;
        wp += tok * tiles_of(i);
    }
    for (int32_t r = threadIdx.x; r < R; r += blockDim.x)
        ws += A.seq_lens[r] - (int64_t)A.suffix_start[r] * kBlockSize;
    wp = block_sum64(wp, red);
    if (threadIdx.x == 0) hdr->prefix_tile_tok_sum = wp;
    wp *= A.Hkv;
    ws = block_sum64(ws, red) * A.Hkv;
    int32_t split_p = A.split_opt, split_s = A.split_opt;
    if (split_p <= 0) {
        // about three items per CTA of the grouped pass, which runs beside the
        // per-request pass on its share of the SMs (the estimate the decode uses)
        const double tp = (double)wp / kPrefixGBsPerSM, tsf = (double)ws / kSuffixGBsPerSM;
        const int32_t np = tp + tsf > 0.0 ? max(1, (int32_t)(0.9 * A.num_sms * tp / (tp + tsf) + 0.5)) : A.num_sms;
        const int64_t t = wp / (int64_t)(3 * min(max(1, A.num_sms), np));
        // no chunk above 4096 tokens: groups of very different lengths need
        // chunks short enough for the CTAs to finish together
        split_p = (int32_t)min((int64_t)4096, max((int64_t)512, (t + 63) / 64 * 64));
    }
    if (split_s <= 0) {
        const int64_t t = ws / (int64_t)(32 * max(1, A.num_sms));
        split_s = (int32_t)min((int64_t)8192, max((int64_t)kMinOwnChunk, (t + 63) / 64 * 64));
    }

    // per-group chunk counts, item offsets, partial bases, member offsets
    const int64_t n_members = block_exclusive_scan(n, [&](int32_t i) { return (int64_t)A.g_nm[i]; },
                                                   A.g_moff, red);
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) {
        // chunks are whole stages of the grouped pass; their count follows
        // from the rounded size, so that every chunk holds tokens (a group
        // folded into its children has none)
        if (folded_in(i)) {
            A.g_chunk[i] = 0;
            A.g_nch[i] = 0;
            continue;
        }
        const int32_t tok = (A.g_b[i] - A.g_wa[i]) * kBlockSize;
        // a group's work up to kWholeItem x the target stays one chunk: an item
        // costs a fixed set-up and epilogue on top of its stages, so one long
        // item beats two short ones unless the balance across CTAs needs them
        const int32_t want = tok <= (int32_t)(kWholeItem * split_p) ? 1 : (tok + split_p - 1) / split_p;
        const int32_t chunk = ((tok + want - 1) / want + kStageTokens - 1) / kStageTokens * kStageTokens;
        A.g_chunk[i] = chunk;
        A.g_nch[i] = (tok + chunk - 1) / chunk;
    }
    __syncthreads();
    const int64_t n_pitems = block_exclusive_scan(
        n, [&](int32_t i) { return (int64_t)A.Hkv * A.g_nch[i] * ((A.g_nm[i] * G + tile_rows - 1) / tile_rows); },
        A.s.g_item_off, red);
    const int64_t n_ppart = block_exclusive_scan(
        n, [&](int32_t i) { return (int64_t)A.Hkv * A.g_nch[i] * A.g_nm[i] * G; }, A.g_part, red);

    // per-request chunks; own-pass items are binned by length, longest first
    int32_t* bins = reinterpret_cast<int32_t*>(red + 64 + 1024);
    for (int32_t b = threadIdx.x; b < kBins; b += blockDim.x) bins[b] = 0;
    __syncthreads();
    for (int32_t r = threadIdx.x; r < R; r += blockDim.x) {
        const int32_t tok = A.seq_lens[r] - A.suffix_start[r] * kBlockSize;
        const int32_t nch = (tok + split_s - 1) / split_s;
        A.s_nch[r] = nch;
        const int32_t chunk = nch ? ((tok + nch - 1) / nch + kBlockSize - 1) / kBlockSize * kBlockSize : 0;
        A.s_chunk[r] = chunk;
        if (nch) {
            const int32_t last = tok - (nch - 1) * chunk;
            atomicAdd(&bins[length_bin(chunk)], A.Hkv * (nch - 1));
            atomicAdd(&bins[length_bin(last)], A.Hkv);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int32_t acc = 0;
        for (int32_t b = kBins - 1; b >= 0; --b) {
            A.bin_cursor[b] = acc;
            acc += bins[b];
        }
    }
    __syncthreads();
    const int32_t split = split_s;
    const int64_t n_sitems = block_exclusive_scan(R, [&](int32_t r) { return (int64_t)A.Hkv * A.s_nch[r]; },
                                                  A.s.s_item_off, red);
    const int64_t n_spart = block_exclusive_scan(
        R, [&](int32_t r) { return (int64_t)A.Hkv * A.s_nch[r] * G; }, A.s_part, red);
    for (int32_t r = threadIdx.x; r < R; r += blockDim.x) A.s_part[r] += (int32_t)n_ppart;
    const int64_t n_chain = block_exclusive_scan(
        R, [&](int32_t r) { return A.flat ? 0 : (int64_t)A.s.n_emit[r]; }, A.chain_off, red);
    int32_t depth = 0;
    for (int32_t r = threadIdx.x; r < R; r += blockDim.x) depth = max(depth, A.flat ? 0 : A.s.n_emit[r]);
    depth = block_max32(depth, red);

    int64_t ptok = 0, stok = 0, ftok = 0;
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) ptok += (int64_t)(A.g_b[i] - A.g_a[i]) * kBlockSize;
    for (int32_t r = threadIdx.x; r < R; r += blockDim.x) {
        stok += A.seq_lens[r] - (int64_t)A.suffix_start[r] * kBlockSize;
        ftok += A.seq_lens[r];
    }
    ptok = block_sum64(ptok, red);
    stok = block_sum64(stok, red);
    ftok = block_sum64(ftok, red);
    if (threadIdx.x == 0) {
        hdr->n_groups = n;
        hdr->n_member_entries = (int32_t)n_members;
        hdr->max_depth = depth;
        hdr->split_tokens = split;
        hdr->prefix_split_tokens = split_p;
        hdr->n_prefix_items = (int32_t)n_pitems;
        hdr->n_suffix_items = (int32_t)n_sitems;
        hdr->n_prefix_partials = (int32_t)n_ppart;
        hdr->n_suffix_partials = (int32_t)n_spart;
        hdr->n_chain_entries = (int32_t)n_chain;
        hdr->prefix_tok_sum = ptok;
        hdr->suffix_tok_sum = stok;
        hdr->fca_kv_tokens = ptok + stok;
        hdr->flat_kv_tokens = ftok;
    }
}

// One CTA per group: sort the member list, then record each member's position
// in its chain.
__global__ void __launch_bounds__(256) k_sort_members(const PlanHeader* hdr, const int32_t* g_moff,
                                                      const int32_t* g_nm, int32_t* members,
                                                      const int32_t* chain_off, const int32_t* chain_g,
                                                      int32_t* chain_pos) {
    extern __shared__ int32_t sm_mem[];
    const int32_t ng = hdr->n_groups;
    for (int32_t g = blockIdx.x; g < ng; g += gridDim.x) {
        const int32_t off = g_moff[g], n = g_nm[g];
        int32_t N = 1;
        while (N < n) N <<= 1;
        for (int32_t i = threadIdx.x; i < N; i += blockDim.x) sm_mem[i] = i < n ? members[off + i] : 0x7FFFFFFF;
        __syncthreads();
        for (int32_t k = 2; k <= N; k <<= 1)
            for (int32_t j = k >> 1; j > 0; j >>= 1) {
                for (int32_t i = threadIdx.x; i < N; i += blockDim.x) {
                    const int32_t p = i ^ j;
                    if (p > i) {
                        const bool up = (i & k) == 0;
                        const int32_t x = sm_mem[i], y = sm_mem[p];
                        if ((x > y) == up) { sm_mem[i] = y; sm_mem[p] = x; }
                    }
                }
                __syncthreads();
            }
        for (int32_t i = threadIdx.x; i < n; i += blockDim.x) {
            const int32_t r = sm_mem[i];
            members[off + i] = r;
            for (int32_t c = chain_off[r]; c < chain_off[r + 1]; ++c)
                if (chain_g[c] == g) chain_pos[c] = i;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------ work lists

// One CTA per group: items (q-tile, chunk, head), heads innermost, over the
// group's work interval [g_wa, g_b) (g_wa is the parent's first block when the
// parent is folded into its children).
__global__ void k_fill_prefix_items(const PlanHeader* hdr, const int32_t* g_wa, const int32_t* g_b,
                                    const int32_t* g_nm, const int32_t* g_moff, const int32_t* g_nch,
                                    const int32_t* g_chunk, const int32_t* g_part, const int32_t* item_off,
                                    const int32_t* members, int32_t G, int32_t Hkv, PrefixItem* items) {
    const int32_t ng = hdr->n_groups;
    for (int32_t g = blockIdx.x; g < ng; g += gridDim.x) {
        const int32_t rows = g_nm[g] * G, tiles = (rows + kPrefixTileRows - 1) / kPrefixTileRows;
        const int32_t nch = g_nch[g], per_head = tiles * nch, split = g_chunk[g];
        const int32_t t0 = g_wa[g] * kBlockSize, t1 = g_b[g] * kBlockSize;
        // heads innermost: the KV heads of one token are neighbours in the cache
        // (one DRAM row holds all of them), so their items should run together
        for (int32_t i = threadIdx.x; i < Hkv * per_head; i += blockDim.x) {
            const int32_t h = i % Hkv, rem = i / Hkv, c = rem % nch, tile = rem / nch;
            PrefixItem it;
            it.moff = g_moff[g];
            it.head = h;
            it.row0 = tile * kPrefixTileRows;
            it.nrows = min(kPrefixTileRows, rows - it.row0);
            it.tok0 = t0 + c * split;
            it.tok1 = min(t1, it.tok0 + split);
            it.bt_row = members[g_moff[g]];
            it.part_row0 = g_part[g] + (h * nch + c) * rows + it.row0;
            items[item_off[g] + i] = it;
        }
    }
}

// Own-pass chunks that any update of a plan can need: request r's own range
// can grow to the table's width past its shared blocks, in chunks of at least
// min_chunk tokens (the update's chunk target never goes below it).
__global__ void __launch_bounds__(1024) k_own_cap(int32_t R, int32_t max_blocks, const int32_t* suffix_start,
                                                  int32_t min_chunk, PlanHeader* hdr) {
    __shared__ int64_t red[64];
    int64_t c = 0;
    for (int32_t r = threadIdx.x; r < R; r += blockDim.x) {
        const int64_t tok = (int64_t)(max_blocks - suffix_start[r]) * kBlockSize;
        c += (tok + min_chunk - 1) / min_chunk;
    }
    c = block_sum64(c, red);
    if (threadIdx.x == 0) hdr->own_chunk_cap = c;
}

// An asynchronous update goes ahead only if every check passed and its own
// work fits the room the plan reserved.
__device__ __forceinline__ bool update_fits(const PlanHeader* hdr, int64_t cap_items, int64_t cap_rows,
                                            int64_t n_ppart) {
    return hdr->status == 0 && hdr->n_suffix_items <= cap_items && n_ppart + hdr->n_suffix_partials <= cap_rows;
}

// gate: null, or the header of an asynchronous update, which writes the
// items only if it fits (update_fits).
__global__ void k_fill_suffix_items(int32_t R, const int32_t* seq_lens, const int32_t* suffix_start,
                                    const int32_t* s_nch, const int32_t* s_chunk, const int32_t* s_part,
                                    int32_t* bin_cursor, int32_t G, int32_t Hkv, SuffixItem* items,
                                    const PlanHeader* gate = nullptr, int64_t cap_items = 0,
                                    int64_t cap_rows = 0, int64_t n_ppart = 0) {
    if (gate && !update_fits(gate, cap_items, cap_rows, n_ppart)) return;
    // one thread per request; the Hkv heads of one chunk take consecutive
    // slots (one DRAM row holds all heads of a token, so they should run together)
    for (int32_t r = blockIdx.x * blockDim.x + threadIdx.x; r < R; r += gridDim.x * blockDim.x) {
        const int32_t nch = s_nch[r], chunk = s_chunk[r];
        const int32_t t0 = suffix_start[r] * kBlockSize, L = seq_lens[r];
        for (int32_t c = 0; c < nch; ++c) {
            const int32_t tok0 = t0 + c * chunk, tok1 = min(L, tok0 + chunk);
            const int32_t pos = atomicAdd(&bin_cursor[length_bin(tok1 - tok0)], Hkv);
            for (int32_t h = 0; h < Hkv; ++h) {
                SuffixItem it;
                it.request = r;
                it.head = h;
                it.tok0 = tok0;
                it.tok1 = tok1;
                it.part_row0 = s_part[r] + (h * nch + c) * G;
                it.pad0 = it.pad1 = it.pad2 = 0;
                items[pos + h] = it;
            }
        }
    }
}

// Per request, its group partials in chain order (the order the merge reads
// them in): group g's chunk c holds member pos's G rows of KV head h at
// g_part + ((h nch + c) nm + pos) G, i.e. x + h y with x = g_part + (c nm +
// pos) G and y = nch nm G.  The first kMergeRec are recorded; m_ng counts all.
__global__ void k_merge_records(int32_t R, int32_t G, const int32_t* chain_off, const int32_t* chain_g,
                                const int32_t* chain_pos, const int32_t* g_nch, const int32_t* g_nm,
                                const int32_t* g_part, int32_t* m_ng, int2* m_rec) {
    for (int32_t r = blockIdx.x * blockDim.x + threadIdx.x; r < R; r += gridDim.x * blockDim.x) {
        int32_t k = 0;
        for (int32_t c = chain_off[r]; c < chain_off[r + 1]; ++c) {
            const int32_t g = chain_g[c], pos = chain_pos[c], nch = g_nch[g], nm = g_nm[g];
            for (int32_t ch = 0; ch < nch; ++ch, ++k)
                if (k < kMergeRec) m_rec[(int64_t)r * kMergeRec + k] = make_int2(g_part[g] + (ch * nm + pos) * G, nch * nm * G);
        }
        m_ng[r] = k;
    }
}

// ------------------------------------------------------------ plan update

// Thread (r, j): the entries of request r's table that its groups read (its
// first suffix_start[r] blocks) must be the plan's, and its length must still
// cover them.
__global__ void k_check_shared(const int32_t* __restrict__ bt_new, const int32_t* __restrict__ sl_new,
                               const int32_t* __restrict__ bt_old, const int32_t* __restrict__ suffix_start,
                               int32_t R, int32_t MB, PlanHeader* hdr) {
    const int64_t total = (int64_t)R * MB;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t r = (int32_t)(i / MB), j = (int32_t)(i % MB);
        const int32_t ss = suffix_start[r];
        if (j == 0 && (int64_t)sl_new[r] < (int64_t)ss * kBlockSize) atomicOr(&hdr->status, kPlanUpdateMismatch);
        if (j < ss && bt_new[i] != bt_old[i]) atomicOr(&hdr->status, kPlanUpdateMismatch);
    }
}

struct UpdateOwnArgs {
    int32_t R, Hkv, G, split_opt, num_sms;
    int64_t n_ppart;               // partial rows of the grouped pass (unchanged)
    const int32_t* seq_lens;       // the new lengths
    const int32_t* suffix_start;   // the plan's
    int32_t* nch;                  // [R] own chunks
    int32_t* chunk;                // [R] tokens per own chunk
    int32_t* part;                 // [R + 1] first partial row of (r, head 0, chunk 0)
    int32_t* s_item_off;           // [R + 1]
    int32_t* bin_cursor;           // [kBins]
    PlanHeader* hdr;
};

// The own-pass half of k_finalize for new lengths over an unchanged forest:
// chunk targets, chunks, length bins, item offsets, partial rows and sizes.
// One CTA of 1024 threads; shared memory: 64 + 1024 int64 of reduction space
// and kBins int32.
__global__ void __launch_bounds__(1024) k_update_own(UpdateOwnArgs A) {
    extern __shared__ int64_t sm_upd[];
    int64_t* red = sm_upd;
    int32_t* bins = reinterpret_cast<int32_t*>(red + 64 + 1024);
    PlanHeader* hdr = A.hdr;
    if (hdr->status) return;   // the update is refused; nothing to compute
    const int32_t R = A.R, G = A.G;
    int64_t ws = 0, ftok = 0;
    for (int32_t r = threadIdx.x; r < R; r += blockDim.x) {
        ws += A.seq_lens[r] - (int64_t)A.suffix_start[r] * kBlockSize;
        ftok += A.seq_lens[r];
    }
    ws = block_sum64(ws, red);
    ftok = block_sum64(ftok, red);
    int32_t split_s = A.split_opt;
    if (split_s <= 0) {
        const int64_t t = ws * A.Hkv / (int64_t)(32 * max(1, A.num_sms));
        split_s = (int32_t)min((int64_t)8192, max((int64_t)kMinOwnChunk, (t + 63) / 64 * 64));
    }
    for (int32_t b = threadIdx.x; b < kBins; b += blockDim.x) bins[b] = 0;
    __syncthreads();
    for (int32_t r = threadIdx.x; r < R; r += blockDim.x) {
        const int32_t tok = A.seq_lens[r] - A.suffix_start[r] * kBlockSize;
        const int32_t nch = (tok + split_s - 1) / split_s;
        const int32_t chunk = nch ? ((tok + nch - 1) / nch + kBlockSize - 1) / kBlockSize * kBlockSize : 0;
        A.nch[r] = nch;
        A.chunk[r] = chunk;
        if (nch) {
            const int32_t last = tok - (nch - 1) * chunk;
            atomicAdd(&bins[length_bin(chunk)], A.Hkv * (nch - 1));
            atomicAdd(&bins[length_bin(last)], A.Hkv);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int32_t acc = 0;
        for (int32_t b = kBins - 1; b >= 0; --b) {
            A.bin_cursor[b] = acc;
            acc += bins[b];
        }
    }
    __syncthreads();
    const int64_t n_sitems = block_exclusive_scan(R, [&](int32_t r) { return (int64_t)A.Hkv * A.nch[r]; },
                                                  A.s_item_off, red);
    const int64_t n_spart = block_exclusive_scan(
        R, [&](int32_t r) { return (int64_t)A.Hkv * A.nch[r] * G; }, A.part, red);
    for (int32_t r = threadIdx.x; r < R; r += blockDim.x) A.part[r] += (int32_t)A.n_ppart;
    if (threadIdx.x == 0) {
        hdr->split_tokens = split_s;
        hdr->n_suffix_items = (int32_t)n_sitems;
        hdr->n_suffix_partials = (int32_t)n_spart;
        hdr->suffix_tok_sum = ws;
        hdr->flat_kv_tokens = ftok;
    }
}

// ------------------------------------------------------------ host helpers

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// The memory pool plans allocate from, one per device, created on first use.
// Its release threshold is unbounded: memory a destroyed plan gave back stays
// mapped in the pool for the next plan instead of being unmapped at the next
// synchronisation, so building a plan per decode step costs no page mapping.
cudaError_t plan_pool(cudaMemPool_t* out) {
    constexpr int kMaxDevices = 64;
    static std::mutex mutex;
    static cudaMemPool_t pools[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mutex);
    if (!pools[dev]) {
        cudaMemPoolProps props{};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        e = cudaMemPoolCreate(&pool, &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = ~uint64_t(0);
        e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) {
            cudaMemPoolDestroy(pool);
            return e;
        }
        pools[dev] = pool;
    }
    *out = pools[dev];
    return cudaSuccess;
}

// Lays arrays out back to back (256-byte aligned) in one allocation from the
// library's plan pool: add() records where each array goes, commit() makes
// the one stream-ordered allocation and sets the pointers.
struct Arena {
    struct Slot {
        void** dst;
        size_t off;
    };
    std::vector<Slot> slots;
    size_t bytes = 0;
    template <typename T>
    size_t add(T** dst, size_t count) {
        const size_t off = bytes;
        slots.push_back({reinterpret_cast<void**>(dst), off});
        bytes += align256(std::max<size_t>(count, 1) * sizeof(T));
        return off;
    }
    void bind(void* base) {
        for (const Slot& sl : slots) *sl.dst = static_cast<uint8_t*>(base) + sl.off;
    }
    cudaError_t commit(cudaStream_t stream, void** base) {
        cudaMemPool_t pool = nullptr;
        cudaError_t e = plan_pool(&pool);
        if (e != cudaSuccess) return e;
        e = cudaMallocFromPoolAsync(base, bytes, pool, stream);
        if (e != cudaSuccess) return e;
        for (const Slot& sl : slots) *sl.dst = static_cast<uint8_t*>(*base) + sl.off;
        return cudaSuccess;
    }
};

// Planner temporaries: one allocation, returned to the pool in stream order.
struct TempArena {
    cudaStream_t stream;
    void* base = nullptr;
    explicit TempArena(cudaStream_t s) : stream(s) {}
    ~TempArena() {
        if (base) cudaFreeAsync(base, stream);
    }
};

// Temporaries of one fca_plan_update: from the plan pool for each update, or
// the plan's own scratch for plans with asynchronous updates.
struct UpdateTemps {
    int32_t* valid = nullptr;
    int32_t* nfull = nullptr;
    PlanHeader* hdr = nullptr;
    int32_t* t_nch = nullptr;
    int32_t* t_chunk = nullptr;
    int32_t* t_part = nullptr;
    int32_t* t_item_off = nullptr;
    int32_t* bin_cursor = nullptr;
    // lays the arrays out in `ta`; returns the bytes that start at zero
    size_t layout(Arena& ta, int32_t R, int32_t num_blocks) {
        ta.add(&valid, num_blocks);
        ta.add(&hdr, 1);
        const size_t zero1 = ta.bytes;
        ta.add(&nfull, R);
        ta.add(&t_nch, R);
        ta.add(&t_chunk, R);
        ta.add(&t_part, R + 1);
        ta.add(&t_item_off, R + 1);
        ta.add(&bin_cursor, kBins);
        return zero1;
    }
};

int grid_for(int64_t work, int threads) {
    int64_t g = (work + threads - 1) / threads;
    return (int)std::max<int64_t>(1, std::min<int64_t>(g, 148 * 16));
}

int32_t next_pow2(int32_t n) {
    int32_t N = 1;
    while (N < n) N <<= 1;
    return N;
}

}  // namespace

#define FCA_CK(x)                                \
    do {                                         \
        if (note_cuda(x) != cudaSuccess) {       \
            (void)cudaGetLastError();            \
            return FCA_ERR_CUDA;                 \
        }                                        \
    } while (0)

// Builds the forest and work lists into P (whose shape fields are set).
// On error the caller frees P.
fca_status plan_build(const int32_t* block_tables, const int32_t* seq_lens, cudaStream_t stream,
                      fca_plan_s* P) {
    const int32_t R = P->R, max_blocks = P->max_blocks, num_blocks = P->num_blocks;
    const int32_t Hkv = P->Hkv, D = P->D, G = P->G;
    const fca_plan_opts& opts = P->opts;
    const bool flat = P->flat;

    // Temporaries.  The arrays that start at zero are laid out back to back
    // (count .. hdr) so that one memset clears them.
    PlanScratch s{};
    int32_t* bin_cursor = nullptr;
    Arena ta;
    ta.add(&s.owner, num_blocks);
    ta.add(&s.pos, num_blocks);
    const size_t zero0 = ta.add(&s.count, num_blocks);
    ta.add(&s.valid, num_blocks);
    ta.add(&s.n_emit, R);
    ta.add(&s.fill, R);
    ta.add(&s.n_raw, 1);
    ta.add(&s.hdr, 1);
    const size_t zero1 = ta.bytes;
    ta.add(&s.nfull, R);
    ta.add(&s.raw, R);
    ta.add(&s.keys, R);
    ta.add(&s.g_item_off, R + 1);
    ta.add(&s.s_item_off, R + 1);
    ta.add(&s.gwork, (size_t)4 * R);
    ta.add(&bin_cursor, kBins);
    TempArena tmp(stream);
    if (ta.commit(stream, &tmp.base) != cudaSuccess) {
        tmp.base = nullptr;
        (void)cudaGetLastError();
        return FCA_ERR_OOM;
    }

    // The plan's arrays whose sizes are known before the planner runs
    // (suffix_start, dev_status and sched start at zero and come first).
    Arena pa;
    pa.add(&P->suffix_start, R);
    pa.add(&P->dev_status, 1);
    pa.add(&P->sched, 4);
    const size_t pzero = pa.bytes;
    pa.add(&P->bt, (size_t)R * max_blocks);
    pa.add(&P->seq_lens, R);
    pa.add(&P->g_a, R);
    pa.add(&P->g_b, R);
    pa.add(&P->g_parent, R);
    pa.add(&P->g_nm, R);
    pa.add(&P->g_moff, R + 1);
    pa.add(&P->g_nch, R);
    pa.add(&P->g_part, R + 1);
    pa.add(&P->s_nch, R);
    pa.add(&P->s_part, R + 1);
    pa.add(&P->g_chunk, R);
    pa.add(&P->s_chunk, R);
    pa.add(&P->g_wa, R);
    pa.add(&P->chain_off, R + 1);
    pa.add(&P->m_ng, R);
    pa.add(&P->m_rec, (size_t)R * kMergeRec);
    {
        void* base = nullptr;
        if (pa.commit(stream, &base) != cudaSuccess) {
            (void)cudaGetLastError();
            return FCA_ERR_OOM;
        }
        P->dev_allocs.push_back(base);
        P->workspace_bytes += pa.bytes;
    }
    s.row_goff = P->chain_off;

    FCA_CK(cudaMemcpyAsync(P->bt, block_tables, sizeof(int32_t) * (size_t)R * max_blocks,
                           cudaMemcpyDeviceToDevice, stream));
    FCA_CK(cudaMemcpyAsync(P->seq_lens, seq_lens, sizeof(int32_t) * R, cudaMemcpyDeviceToDevice, stream));
    FCA_CK(cudaMemsetAsync(s.owner, 0x7F, sizeof(int32_t) * (size_t)num_blocks, stream));
    FCA_CK(cudaMemsetAsync(s.pos, 0xFF, sizeof(int32_t) * (size_t)num_blocks, stream));
    FCA_CK(cudaMemsetAsync(static_cast<uint8_t*>(tmp.base) + zero0, 0, zero1 - zero0, stream));
    FCA_CK(cudaMemsetAsync(P->suffix_start, 0, pzero, stream));

    const int64_t cells = (int64_t)R * max_blocks;
    k_validate<<<grid_for(cells, 256), 256, 0, stream>>>(P->bt, max_blocks, P->seq_lens, R, num_blocks, s.nfull,
                                                         s.valid, s.hdr);
    k_unique_tokens<<<grid_for(num_blocks, 256), 256, 0, stream>>>(s.valid, num_blocks, s.hdr);
    FCA_CK(cudaGetLastError());

    RowArgs ra{};
    size_t row_smem = 0;
    const int row_grid = std::min(R, 148 * 8);
    if (!flat) {
        k_block_keys<<<grid_for(cells, 256), 256, 0, stream>>>(P->bt, max_blocks, R, s.nfull, s.owner, s.count,
                                                               s.pos, s.hdr);
        k_check_chain<<<grid_for(cells, 256), 256, 0, stream>>>(P->bt, max_blocks, R, s.nfull, s.owner, s.hdr);
        ra.bt = P->bt;
        ra.MB = max_blocks;
        ra.R = R;
        ra.G = G;
        ra.min_group_size = opts.min_group_size;
        ra.min_shared_blocks = opts.min_shared_blocks;
        ra.min_saved_blocks = opts.min_saved_blocks;
        ra.pass = 0;
        ra.nfull = s.nfull;
        ra.owner = s.owner;
        ra.count = s.count;
        ra.s = s;
        ra.suffix_start = P->suffix_start;
        // the fallback keeps 8-byte sort keys and two int32 arrays per request
        row_smem = R <= kMaxRequestsFallback ? (size_t)next_pow2(R) * 16 : 0;
        FCA_CK(cudaFuncSetAttribute(k_row_runs, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)row_smem));
        k_row_runs<<<row_grid, 256, row_smem, stream>>>(ra);
        FCA_CK(cudaGetLastError());
    }

    FinalizeArgs fa{};
    fa.s = s;
    fa.R = R;
    fa.G = G;
    fa.Hkv = Hkv;
    fa.split_opt = opts.split_tokens;
    fa.flat = flat ? 1 : 0;
    fa.seq_lens = P->seq_lens;
    fa.suffix_start = P->suffix_start;
    fa.g_a = P->g_a;
    fa.g_b = P->g_b;
    fa.g_parent = P->g_parent;
    fa.g_nm = P->g_nm;
    fa.g_moff = P->g_moff;
    fa.g_nch = P->g_nch;
    fa.g_part = P->g_part;
    fa.s_nch = P->s_nch;
    fa.s_part = P->s_part;
    fa.chain_off = P->chain_off;
    fa.g_chunk = P->g_chunk;
    fa.s_chunk = P->s_chunk;
    fa.g_wa = P->g_wa;
    fa.bin_cursor = bin_cursor;
    {
        int dev = 0;
        cudaGetDevice(&dev);
        fa.num_sms = 148;
        cudaDeviceGetAttribute(&fa.num_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const size_t fin_smem = (size_t)next_pow2(R) * 8 + (64 + 1024) * 8 + kBins * 4;
    FCA_CK(cudaFuncSetAttribute(k_finalize, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fin_smem));
    k_finalize<<<1, 1024, fin_smem, stream>>>(fa);
    FCA_CK(cudaGetLastError());

    if (P->async_update) {
        const int32_t min_chunk = opts.split_tokens > 0 ? opts.split_tokens : kMinOwnChunk;
        k_own_cap<<<1, 1024, 0, stream>>>(R, max_blocks, P->suffix_start, min_chunk, s.hdr);
        FCA_CK(cudaGetLastError());
    }

    // the one synchronisation: sizes of the forest and of the work lists
    FCA_CK(cudaMemcpyAsync(&P->hdr, s.hdr, sizeof(PlanHeader), cudaMemcpyDeviceToHost, stream));
    FCA_CK(cudaStreamSynchronize(stream));
    const PlanHeader& H = P->hdr;
    if (H.status & kPlanBadSeqLen) return FCA_ERR_INVALID_ARG;
    if (H.status & kPlanBadBlockId) return FCA_ERR_BAD_BLOCK_ID;
    if (H.status & kPlanTooManyGroups) return FCA_ERR_UNSUPPORTED;
    if ((H.status & kPlanInconsistent) && R > kMaxRequestsFallback) return FCA_ERR_UNSUPPORTED;
    // own-pass room: what this plan needs, or (asynchronous updates) what any update can
    const int64_t cap_items =
        P->async_update ? std::max<int64_t>(H.n_suffix_items, (int64_t)Hkv * H.own_chunk_cap) : H.n_suffix_items;
    const int64_t n_part = (int64_t)H.n_prefix_partials + cap_items * G;
    if (n_part >= (int64_t)INT32_MAX / 2) return FCA_ERR_UNSUPPORTED;

    // the arrays sized by the planner
    Arena wa;
    wa.add(&P->members, H.n_member_entries);
    wa.add(&P->chain_g, H.n_chain_entries);
    wa.add(&P->chain_pos, H.n_chain_entries);
    wa.add(&P->prefix_items, H.n_prefix_items);
    wa.add(&P->suffix_items, cap_items);
    wa.add(&P->part_lse, n_part);
    wa.add(&P->part_o, (size_t)n_part * D);
    if (P->async_update) {
        UpdateTemps T;
        Arena probe;
        T.layout(probe, R, num_blocks);
        wa.add(reinterpret_cast<uint8_t**>(&P->upd_scratch), probe.bytes);
    }
    {
        void* base = nullptr;
        if (wa.commit(stream, &base) != cudaSuccess) {
            (void)cudaGetLastError();
            return FCA_ERR_OOM;
        }
        P->dev_allocs.push_back(base);
        P->workspace_bytes += wa.bytes;
        P->cap_suffix_items = cap_items;
        P->cap_partials = n_part;
    }
    if (P->async_update)   // the per-request pass's item count, read on the device
        FCA_CK(cudaMemcpyAsync(P->sched + 2, &P->hdr.n_suffix_items, sizeof(int32_t), cudaMemcpyHostToDevice,
                               stream));

    if (!flat && H.n_groups > 0) {
        ra.pass = 1;
        ra.keys = s.keys;
        ra.g_moff = P->g_moff;
        ra.members = P->members;
        ra.chain_g = P->chain_g;
        ra.err = P->dev_status;
        k_row_runs<<<row_grid, 256, row_smem, stream>>>(ra);
        FCA_CK(cudaGetLastError());
        const size_t mem_smem = (size_t)next_pow2(R) * 4;
        FCA_CK(cudaFuncSetAttribute(k_sort_members, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mem_smem));
        k_sort_members<<<std::min(H.n_groups, 148 * 4), 256, mem_smem, stream>>>(
            s.hdr, P->g_moff, P->g_nm, P->members, P->chain_off, P->chain_g, P->chain_pos);
        k_fill_prefix_items<<<std::min(H.n_groups, 148 * 4), 256, 0, stream>>>(
            s.hdr, P->g_wa, P->g_b, P->g_nm, P->g_moff, P->g_nch, P->g_chunk, P->g_part, s.g_item_off, P->members,
            G, Hkv, P->prefix_items);
        FCA_CK(cudaGetLastError());
    }
    if (H.n_suffix_items > 0) {
        k_fill_suffix_items<<<grid_for(R, 128), 128, 0, stream>>>(
            R, P->seq_lens, P->suffix_start, P->s_nch, P->s_chunk, P->s_part, bin_cursor, G, Hkv, P->suffix_items);
        FCA_CK(cudaGetLastError());
    }
    k_merge_records<<<grid_for(R, 128), 128, 0, stream>>>(R, G, P->chain_off, P->chain_g, P->chain_pos, P->g_nch,
                                                          P->g_nm, P->g_part, P->m_ng, P->m_rec);
    FCA_CK(cudaGetLastError());
    return FCA_OK;   // temporaries go back to the pool in stream order
}

// Applies an asynchronous update on the device: the new tables, lengths and
// own-pass arrays replace the plan's, and the per-request pass's item count
// (sched[2]) is set, if the update fits; otherwise nothing changes and the
// plan's status word records kErrUpdateRefused.
struct UpdateApplyArgs {
    const PlanHeader* hdr;
    int64_t cap_items, cap_rows, n_ppart, cells;
    int32_t R;
    const int32_t* bt_new;
    const int32_t* sl_new;
    const int32_t* t_nch;
    const int32_t* t_chunk;
    const int32_t* t_part;
    int32_t* bt;
    int32_t* seq_lens;
    int32_t* s_nch;
    int32_t* s_chunk;
    int32_t* s_part;
    int32_t* sched;
    int32_t* err;
};

__global__ void k_update_apply(UpdateApplyArgs A) {
    if (!update_fits(A.hdr, A.cap_items, A.cap_rows, A.n_ppart)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(A.err, kErrUpdateRefused);
        return;
    }
    const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x, step = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = t0; i < A.cells; i += step) A.bt[i] = A.bt_new[i];
    for (int64_t r = t0; r < A.R; r += step) {
        A.seq_lens[r] = A.sl_new[r];
        A.s_nch[r] = A.t_nch[r];
        A.s_chunk[r] = A.t_chunk[r];
    }
    for (int64_t r = t0; r <= A.R; r += step) A.s_part[r] = A.t_part[r];
    if (t0 == 0) A.sched[2] = A.hdr->n_suffix_items;
}

// Next decode step of the same batch: new lengths (and tables grown past the
// blocks the plan's groups read) over the plan's forest.  Everything is
// checked before the plan changes; on an error return it is as it was.
fca_status plan_update(const int32_t* block_tables, const int32_t* seq_lens, cudaStream_t stream,
                       fca_plan_s* P) {
    const int32_t R = P->R, max_blocks = P->max_blocks, num_blocks = P->num_blocks;
    const int32_t Hkv = P->Hkv, D = P->D, G = P->G;

    UpdateTemps T;
    Arena ta;
    const size_t zero1 = T.layout(ta, R, num_blocks);
    int32_t* valid = T.valid;
    int32_t* nfull = T.nfull;
    PlanHeader* hdr = T.hdr;
    int32_t* t_nch = T.t_nch;
    int32_t* t_chunk = T.t_chunk;
    int32_t* t_part = T.t_part;
    int32_t* t_item_off = T.t_item_off;
    int32_t* bin_cursor = T.bin_cursor;
    TempArena tmp(stream);
    void* tbase = nullptr;
    if (P->async_update) {
        // the plan's own scratch (no allocation, so that the update can be
        // captured in a CUDA graph along with the decode)
        ta.bind(P->upd_scratch);
        tbase = P->upd_scratch;
    } else {
        if (ta.commit(stream, &tmp.base) != cudaSuccess) {
            tmp.base = nullptr;
            (void)cudaGetLastError();
            return FCA_ERR_OOM;
        }
        tbase = tmp.base;
    }
    valid = T.valid;
    nfull = T.nfull;
    hdr = T.hdr;
    t_nch = T.t_nch;
    t_chunk = T.t_chunk;
    t_part = T.t_part;
    t_item_off = T.t_item_off;
    bin_cursor = T.bin_cursor;
    FCA_CK(cudaMemsetAsync(tbase, 0, zero1, stream));
    const int64_t cells = (int64_t)R * max_blocks;
    k_validate<<<grid_for(cells, 256), 256, 0, stream>>>(block_tables, max_blocks, seq_lens, R, num_blocks, nfull,
                                                          valid, hdr);
    k_check_shared<<<grid_for(cells, 256), 256, 0, stream>>>(block_tables, seq_lens, P->bt, P->suffix_start, R,
                                                             max_blocks, hdr);
    k_unique_tokens<<<grid_for(num_blocks, 256), 256, 0, stream>>>(valid, num_blocks, hdr);
    FCA_CK(cudaGetLastError());
    UpdateOwnArgs ua{};
    ua.R = R;
    ua.Hkv = Hkv;
    ua.G = G;
    ua.split_opt = P->opts.split_tokens;
    {
        int dev = 0;
        cudaGetDevice(&dev);
        ua.num_sms = 148;
        cudaDeviceGetAttribute(&ua.num_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    ua.n_ppart = P->hdr.n_prefix_partials;
    ua.seq_lens = seq_lens;
    ua.suffix_start = P->suffix_start;
    ua.nch = t_nch;
    ua.chunk = t_chunk;
    ua.part = t_part;
    ua.s_item_off = t_item_off;
    ua.bin_cursor = bin_cursor;
    ua.hdr = hdr;
    const size_t upd_smem = (64 + 1024) * 8 + kBins * 4;
    k_update_own<<<1, 1024, upd_smem, stream>>>(ua);
    FCA_CK(cudaGetLastError());

    if (P->async_update) {
        // checked, sized and applied on the device; no host synchronisation
        UpdateApplyArgs ap{};
        ap.hdr = hdr;
        ap.cap_items = P->cap_suffix_items;
        ap.cap_rows = P->cap_partials;
        ap.n_ppart = P->hdr.n_prefix_partials;
        ap.cells = cells;
        ap.R = R;
        ap.bt_new = block_tables;
        ap.sl_new = seq_lens;
        ap.t_nch = t_nch;
        ap.t_chunk = t_chunk;
        ap.t_part = t_part;
        ap.bt = P->bt;
        ap.seq_lens = P->seq_lens;
        ap.s_nch = P->s_nch;
        ap.s_chunk = P->s_chunk;
        ap.s_part = P->s_part;
        ap.sched = P->sched;
        ap.err = P->dev_status;
        k_update_apply<<<grid_for(cells, 256), 256, 0, stream>>>(ap);
        k_fill_suffix_items<<<grid_for(R, 128), 128, 0, stream>>>(R, P->seq_lens, P->suffix_start, P->s_nch,
                                                                  P->s_chunk, P->s_part, bin_cursor, G, Hkv,
                                                                  P->suffix_items, hdr, P->cap_suffix_items,
                                                                  P->cap_partials, P->hdr.n_prefix_partials);
        FCA_CK(cudaGetLastError());
        return FCA_OK;   // temporaries go back to the pool in stream order
    }

    PlanHeader H{};
    FCA_CK(cudaMemcpyAsync(&H, hdr, sizeof(PlanHeader), cudaMemcpyDeviceToHost, stream));
    FCA_CK(cudaStreamSynchronize(stream));
    if (H.status & kPlanBadSeqLen) return FCA_ERR_INVALID_ARG;
    if (H.status & kPlanBadBlockId) return FCA_ERR_BAD_BLOCK_ID;
    if (H.status & kPlanUpdateMismatch) return FCA_ERR_INVALID_ARG;
    const int64_t n_part = (int64_t)P->hdr.n_prefix_partials + H.n_suffix_partials;
    if (n_part >= (int64_t)INT32_MAX / 2) return FCA_ERR_UNSUPPORTED;

    // more own work than the plan has room for: a new block for the own-pass
    // items and every partial row (the grouped pass's rows are rewritten by
    // each decode, so nothing needs copying)
    if (H.n_suffix_items > P->cap_suffix_items || n_part > P->cap_partials) {
        const int64_t items = std::max<int64_t>(H.n_suffix_items, P->cap_suffix_items) * 5 / 4 + 64;
        const int64_t rows = std::max<int64_t>(n_part, P->cap_partials) * 5 / 4 + 64;
        SuffixItem* n_items = nullptr;
        float* n_lse = nullptr;
        float* n_o = nullptr;
        Arena na;
        na.add(&n_items, (size_t)items);
        na.add(&n_lse, (size_t)rows);
        na.add(&n_o, (size_t)rows * D);
        void* base = nullptr;
        if (na.commit(stream, &base) != cudaSuccess) {
            (void)cudaGetLastError();
            return FCA_ERR_OOM;
        }
        P->dev_allocs.push_back(base);
        P->workspace_bytes += na.bytes;
        P->suffix_items = n_items;
        P->part_lse = n_lse;
        P->part_o = n_o;
        P->cap_suffix_items = items;
        P->cap_partials = rows;
    }

    // apply: the new tables and lengths, the own-pass arrays, the item list
    FCA_CK(cudaMemcpyAsync(P->bt, block_tables, (size_t)cells * sizeof(int32_t), cudaMemcpyDeviceToDevice, stream));
    FCA_CK(cudaMemcpyAsync(P->seq_lens, seq_lens, (size_t)R * sizeof(int32_t), cudaMemcpyDeviceToDevice, stream));
    FCA_CK(cudaMemcpyAsync(P->s_nch, t_nch, (size_t)R * sizeof(int32_t), cudaMemcpyDeviceToDevice, stream));
    FCA_CK(cudaMemcpyAsync(P->s_chunk, t_chunk, (size_t)R * sizeof(int32_t), cudaMemcpyDeviceToDevice, stream));
    FCA_CK(cudaMemcpyAsync(P->s_part, t_part, (size_t)(R + 1) * sizeof(int32_t), cudaMemcpyDeviceToDevice, stream));
    if (H.n_suffix_items > 0) {
        k_fill_suffix_items<<<grid_for(R, 128), 128, 0, stream>>>(R, P->seq_lens, P->suffix_start, P->s_nch,
                                                                  P->s_chunk, P->s_part, bin_cursor, G, Hkv,
                                                                  P->suffix_items);
        FCA_CK(cudaGetLastError());
    }
    PlanHeader& PH = P->hdr;
    PH.split_tokens = H.split_tokens;
    PH.n_suffix_items = H.n_suffix_items;
    PH.n_suffix_partials = H.n_suffix_partials;
    PH.suffix_tok_sum = H.suffix_tok_sum;
    PH.flat_kv_tokens = H.flat_kv_tokens;
    PH.unique_kv_tokens = H.unique_kv_tokens;
    PH.fca_kv_tokens = PH.prefix_tok_sum + H.suffix_tok_sum;
    return FCA_OK;   // temporaries go back to the pool in stream order
}

#undef FCA_CK

}  // namespace fca
