// fca_paged_decode_static: the flat paged decode (every request over its
// whole block table, split-KV, then the log-sum-exp merge) for callers that
// cannot allocate device memory, e.g. code running inside a serving engine
// whose device memory is all handed out by its own pool, or code that must
// not call the CUDA allocator while a stream is being recorded.
//
// The per-request kernel and the merge kernel are the ones fca_flat_decode
// runs ("ZoRRo Inference & Forest Cascade Attention", "Core Mechanism" step 2,
// second bullet, and step 3).  What differs is where their work list and
// partial results live: not in a plan's cudaMalloc'd workspace but in one
// fixed array of this library (g_scratch below), sized at build time.  A
// small kernel builds the work list there from the device block tables and
// sequence lengths, so the call needs neither a plan nor a host round trip.
#include <algorithm>
#include <mutex>

#include <cuda_bf16.h>

#include "fca_internal.h"

namespace fca {

cudaError_t launch_suffix_devcount(const fca_plan_s* P, const void* q, const CUtensorMap& tk,
                                   const CUtensorMap& tv, float scale, cudaStream_t stream);
cudaError_t launch_merge(const fca_plan_s* P, void* out, float* lse, bool after_pass, cudaStream_t stream);

static_assert(FCA_STATIC_SCRATCH_BYTES == kStaticScratchBytes, "fca.h and the library disagree on the scratch size");

namespace {

// The scratch: one per device, allocated by the CUDA runtime when it loads
// this library's kernels on that device (zero-filled then).
__device__ __align__(256) uint8_t g_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_addr_mutex;
void* g_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device, looked up once per
// device (the first call on a device does the lookup, which may load the
// module there).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_addr_mutex);
    if (!g_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Byte offsets of the scratch's parts for R requests and C chunks a request.
struct ScratchLayout {
    size_t sched, err, chain_off, s_nch, s_part, items, part_lse, part_o, total;
    ScratchLayout(int64_t R, int64_t Hq, int64_t Hkv, int64_t D, int64_t C) {
        sched = 0;                         // int32 [4]: next item, warps done, item count, unused
        err = 64;                          // int32: error word when the caller passes none
        chain_off = 256;                   // int32 [R + 1], all zero: no groups
        s_nch = chain_off + align256(4 * (R + 1));
        s_part = s_nch + align256(4 * R);
        items = s_part + align256(4 * R);
        part_lse = items + align256(sizeof(SuffixItem) * R * Hkv * C);
        part_o = part_lse + align256(4 * R * Hq * C);
        total = part_o + align256(4 * R * Hq * C * D);
    }
};

struct FillArgs {
    const int32_t* bt;
    const int32_t* seq_lens;
    int32_t R, max_blocks, num_blocks, Hq, Hkv, G, C, S;
    int32_t* sched;
    int32_t* err;
    int32_t* chain_off;
    int32_t* s_nch;
    int32_t* s_part;
    SuffixItem* items;
};

// One warp per request: check its length and the block ids it uses, then
// append its (chunk, KV head) items to the list.  Request r owns partial rows
// [r Hq C, (r + 1) Hq C); its item (h, c) writes the G rows starting at
// r Hq C + (h nsc + c) G, the order the merge reads them in.
__global__ void __launch_bounds__(256) k_static_fill(FillArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t r = blockIdx.x * 8 + warp;
    if (r >= a.R) return;
    const int32_t L = a.seq_lens[r];
    const bool len_ok = L >= 1 && (int64_t)L <= (int64_t)a.max_blocks * kBlockSize;
    const int32_t nb = len_ok ? (L + kBlockSize - 1) / kBlockSize : 0;
    bool bad = false;
    for (int32_t j = lane; j < nb; j += 32) {
        const int32_t b = a.bt[(int64_t)r * a.max_blocks + j];
        bad |= b < 0 || b >= a.num_blocks;
    }
    bad = __any_sync(0xffffffffu, bad);
    const int32_t nsc = (len_ok && !bad) ? (L + a.S - 1) / a.S : 0;
    const int32_t part0 = r * a.Hq * a.C;
    int32_t base = 0;
    if (lane == 0) {
        if (!len_ok) atomicOr(a.err, kErrStaticSeqLen);
        if (bad) atomicOr(a.err, kErrStaticBlockId);
        a.s_nch[r] = nsc;
        a.s_part[r] = part0;
        a.chain_off[r + 1] = 0;
        if (r == 0) a.chain_off[0] = 0;
        if (nsc > 0) base = atomicAdd(a.sched + 2, nsc * a.Hkv);
    }
    base = __shfl_sync(0xffffffffu, base, 0);
    for (int32_t i = lane; i < nsc * a.Hkv; i += 32) {
        const int32_t c = i / a.Hkv, h = i % a.Hkv;
        SuffixItem it;
        it.request = r;
        it.head = h;
        it.tok0 = c * a.S;
        it.tok1 = min((c + 1) * a.S, L);
        it.part_row0 = part0 + (h * nsc + c) * a.G;
        it.pad0 = it.pad1 = it.pad2 = 0;
        a.items[base + i] = it;
    }
}

}  // namespace
}  // namespace fca

using namespace fca;

extern "C" fca_status fca_paged_decode_static(const void* q, const void* k_cache, const void* v_cache,
                                              const int32_t* block_tables, int32_t max_blocks,
                                              const int32_t* seq_lens, int32_t num_requests,
                                              int32_t num_blocks, int32_t num_q_heads, int32_t num_kv_heads,
                                              int32_t head_dim, void* out, float* lse, float scale,
                                              int32_t* dev_status, void* stream) {
    if (!q || !k_cache || !v_cache || !block_tables || !seq_lens || !out || num_requests < 0 || max_blocks < 1 ||
        num_blocks < 1 || num_q_heads < 1 || num_kv_heads < 1 || num_q_heads % num_kv_heads != 0 ||
        !(scale > 0.f) || !(scale < INFINITY))
        return FCA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) || (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u) || (reinterpret_cast<uintptr_t>(dev_status) & 3u))
        return FCA_ERR_INVALID_ARG;
    if ((head_dim != 64 && head_dim != 128) || num_q_heads / num_kv_heads > kMaxGqa ||
        (int64_t)num_blocks * kBlockSize > INT32_MAX || (int64_t)max_blocks * kBlockSize > INT32_MAX)
        return FCA_ERR_UNSUPPORTED;
    if (num_requests == 0) return FCA_OK;

    const int64_t R = num_requests, Hq = num_q_heads, Hkv = num_kv_heads, D = head_dim;
    const int64_t Lmax = (int64_t)max_blocks * kBlockSize;
    if (ScratchLayout(R, Hq, Hkv, D, 1).total > kStaticScratchBytes) return FCA_ERR_TOO_LARGE;

    // Chunks per request: enough items for two per warp slot of the GPU, no
    // chunk under 256 tokens, and no more than the scratch holds.
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (2 * (int64_t)sms * 8 + R * Hkv - 1) / (R * Hkv);
    int64_t C = std::max<int64_t>(1, std::min(want, (Lmax + 255) / 256));
    while (C > 1 && ScratchLayout(R, Hq, Hkv, D, C).total > kStaticScratchBytes) --C;
    const int64_t S = ((Lmax + C - 1) / C + kBlockSize - 1) / kBlockSize * kBlockSize;
    C = (Lmax + S - 1) / S;
    const ScratchLayout lay(R, Hq, Hkv, D, C);

    void* base = nullptr;
    if (note_cuda(scratch_address(&base)) != cudaSuccess) return FCA_ERR_CUDA;
    uint8_t* sb = static_cast<uint8_t*>(base);
    CUtensorMap tk, tv;
    if (!make_cache_map(&tk, k_cache, num_blocks, num_kv_heads, head_dim) ||
        !make_cache_map(&tv, v_cache, num_blocks, num_kv_heads, head_dim))
        return FCA_ERR_CUDA;

    // A view of the scratch in the shape the two kernels' launchers read.
    fca_plan_s V;
    V.R = num_requests;
    V.max_blocks = max_blocks;
    V.block_size = kBlockSize;
    V.num_blocks = num_blocks;
    V.Hq = num_q_heads;
    V.Hkv = num_kv_heads;
    V.D = head_dim;
    V.G = num_q_heads / num_kv_heads;
    V.flat = true;
    V.hdr.n_suffix_items = (int32_t)(R * Hkv * C);   // bound; the kernel reads the count it was given
    V.bt = const_cast<int32_t*>(block_tables);
    V.seq_lens = const_cast<int32_t*>(seq_lens);
    V.sched = reinterpret_cast<int32_t*>(sb + lay.sched);
    V.dev_status = dev_status ? dev_status : reinterpret_cast<int32_t*>(sb + lay.err);
    V.chain_off = reinterpret_cast<int32_t*>(sb + lay.chain_off);
    V.s_nch = reinterpret_cast<int32_t*>(sb + lay.s_nch);
    V.s_part = reinterpret_cast<int32_t*>(sb + lay.s_part);
    V.suffix_items = reinterpret_cast<SuffixItem*>(sb + lay.items);
    V.part_lse = reinterpret_cast<float*>(sb + lay.part_lse);
    V.part_o = reinterpret_cast<float*>(sb + lay.part_o);

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the three counters start at zero on every call
    if (note_cuda(cudaMemsetAsync(V.sched, 0, 4 * sizeof(int32_t), s)) != cudaSuccess) return FCA_ERR_CUDA;
    FillArgs f;
    f.bt = block_tables;
    f.seq_lens = seq_lens;
    f.R = num_requests;
    f.max_blocks = max_blocks;
    f.num_blocks = num_blocks;
    f.Hq = num_q_heads;
    f.Hkv = num_kv_heads;
    f.G = V.G;
    f.C = (int32_t)C;
    f.S = (int32_t)S;
    f.sched = V.sched;
    f.err = V.dev_status;
    f.chain_off = V.chain_off;
    f.s_nch = V.s_nch;
    f.s_part = V.s_part;
    f.items = V.suffix_items;
    k_static_fill<<<(num_requests + 7) / 8, 256, 0, s>>>(f);
    if (note_cuda(cudaGetLastError()) != cudaSuccess) return FCA_ERR_CUDA;
    if (note_cuda(launch_suffix_devcount(&V, q, tk, tv, scale, s)) != cudaSuccess) return FCA_ERR_CUDA;
    if (note_cuda(launch_merge(&V, out, lse, false, s)) != cudaSuccess) return FCA_ERR_CUDA;
    return FCA_OK;
}
