// C ABI of libfca_b200 (declared in include/fca.h): argument checks, plan
// lifetime, TMA descriptors and the launch order of one decode step.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "fca_internal.h"

namespace fca {
fca_status plan_build(const int32_t* block_tables, const int32_t* seq_lens, cudaStream_t stream, fca_plan_s* P);
fca_status plan_update(const int32_t* block_tables, const int32_t* seq_lens, cudaStream_t stream, fca_plan_s* P);
cudaError_t launch_prefix(const fca_plan_s* P, const void* q, const CUtensorMap& tk, const CUtensorMap& tv,
                          float scale, int max_ctas, cudaStream_t stream);
cudaError_t launch_suffix(const fca_plan_s* P, const void* q, const CUtensorMap& tk, const CUtensorMap& tv,
                          float scale, bool beside, cudaStream_t stream);
cudaError_t launch_merge(const fca_plan_s* P, void* out, float* lse, bool after_pass, cudaStream_t stream);

namespace {
thread_local cudaError_t g_last_error = cudaSuccess;
}  // namespace

cudaError_t note_cuda(cudaError_t e) {
    if (e != cudaSuccess) g_last_error = e;
    return e;
}

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            (void)cudaGetLastError();
    });
    return fn;
}

}  // namespace

// Cache [num_blocks * 16 tokens][Hkv][D] bf16 viewed as a 3-D tensor
// (innermost first: D, Hkv, tokens); box = 64 head-dim elements x 1 head x
// 16 tokens (one paged block of one head, one 128-byte swizzle atom wide).
bool make_cache_map(CUtensorMap* map, const void* base, int32_t num_blocks, int32_t Hkv, int32_t D) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)num_blocks * kBlockSize};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kBlockSize};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Makes a plan's device current for one call and restores the caller's
// device afterwards (a no-op when it is current already).
struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev) {
        int cur = 0;
        if (cudaGetDevice(&cur) == cudaSuccess && cur != dev && cudaSetDevice(dev) == cudaSuccess) prev = cur;
        (void)cudaGetLastError();
    }
    ~DeviceGuard() {
        if (prev >= 0) cudaSetDevice(prev);
    }
};

}  // namespace fca

using namespace fca;

extern "C" {

void fca_plan_opts_default(fca_plan_opts* opts) {
    if (!opts) return;
    opts->min_group_size = 2;
    opts->min_shared_blocks = 1;
    opts->min_saved_blocks = kDefaultMinSavedBlocks;
    opts->split_tokens = 0;
    opts->flags = 0;
}

fca_status fca_plan_destroy(fca_plan_t plan) {
    if (!plan) return FCA_OK;
    DeviceGuard dg(plan->device);
    // the plan's memory goes back to the library's pool once nothing that may
    // read it is still running
    cudaDeviceSynchronize();
    for (void* p : plan->dev_allocs) cudaFreeAsync(p, cudaStreamLegacy);
    cudaStreamSynchronize(cudaStreamLegacy);
    (void)cudaGetLastError();
    delete plan;
    return FCA_OK;
}

fca_status fca_plan(const int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens, int32_t num_requests,
                    int32_t block_size, int32_t num_blocks, int32_t num_q_heads, int32_t num_kv_heads,
                    int32_t head_dim, const fca_plan_opts* opts, fca_plan_t* out_plan, void* stream) {
    if (!out_plan) return FCA_ERR_INVALID_ARG;
    *out_plan = nullptr;
    if (!block_tables || !seq_lens || num_requests < 1 || max_blocks < 1 || num_blocks < 1 || num_q_heads < 1 ||
        num_kv_heads < 1 || num_q_heads % num_kv_heads != 0)
        return FCA_ERR_INVALID_ARG;
    if (block_size != kBlockSize || (head_dim != 64 && head_dim != 128) || num_q_heads / num_kv_heads > kMaxGqa ||
        num_requests > kMaxRequests || max_blocks > (1 << 20) || (int64_t)num_blocks * kBlockSize > INT32_MAX)
        return FCA_ERR_UNSUPPORTED;
    fca_plan_opts o;
    fca_plan_opts_default(&o);
    if (opts) o = *opts;
    if (o.min_group_size < 2 || o.min_shared_blocks < 1 || o.min_saved_blocks < 0 || o.split_tokens < 0 ||
        o.split_tokens % 64 != 0)
        return FCA_ERR_INVALID_ARG;
    fca_plan_s* P = new (std::nothrow) fca_plan_s();
    if (!P) return FCA_ERR_OOM;
    cudaGetDevice(&P->device);
    P->R = num_requests;
    P->max_blocks = max_blocks;
    P->block_size = block_size;
    P->num_blocks = num_blocks;
    P->Hq = num_q_heads;
    P->Hkv = num_kv_heads;
    P->D = head_dim;
    P->G = num_q_heads / num_kv_heads;
    P->opts = o;
    P->flat = (o.flags & FCA_PLAN_FLAT) != 0;
    P->async_update = (o.flags & FCA_PLAN_ASYNC_UPDATE) != 0;
    const fca_status st = plan_build(block_tables, seq_lens, static_cast<cudaStream_t>(stream), P);
    if (st != FCA_OK) {
        fca_plan_destroy(P);
        return st;
    }
    *out_plan = P;
    return FCA_OK;
}

fca_status fca_plan_update(fca_plan_t plan, const int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens,
                           int32_t num_requests, void* stream) {
    if (!plan || !block_tables || !seq_lens) return FCA_ERR_INVALID_ARG;
    if (max_blocks != plan->max_blocks || num_requests != plan->R) return FCA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return FCA_ERR_INVALID_ARG;
    DeviceGuard dg(plan->device);
    return plan_update(block_tables, seq_lens, static_cast<cudaStream_t>(stream), plan);
}

// SMs given to the grouped pass when it runs beside the per-request pass:
// 1.15 x the share that would make both finish together at their measured
// per-SM rates (kPrefixGBsPerSM, kSuffixGBsPerSM), the grouped pass's work
// counted in tile-tokens, then trimmed to the fewest SMs that still take its
// items in the same number of rounds.  The per-request pass starts on the
// other SMs and takes over each SM the grouped pass gives up, so the grouped
// pass must not be the last to finish: of 0.8, 0.9, 1.0 and 1.15, 1.15 gave
// the fastest steps on the llama8b, longctx and mixed workloads (forest: the
// same split from 0.9 up).
static int prefix_share(const fca_plan_s* P, int sms) {
    const double tp = (double)P->hdr.prefix_tile_tok_sum / kPrefixGBsPerSM;
    const double ts = (double)P->hdr.suffix_tok_sum / kSuffixGBsPerSM;
    int n = (int)(1.15 * sms * tp / (tp + ts) + 0.5);
    n = std::max(1, std::min(sms - 1, n));
    const int items = P->hdr.n_prefix_items;
    const int rounds = (items + n - 1) / n;
    return std::max(1, std::min(n, (items + rounds - 1) / rounds));
}

static fca_status decode_impl(const void* q, const void* k_cache, const void* v_cache, fca_plan_t plan, void* out,
                              float* lse, float scale, void* stream) {
    if (!plan || !q || !k_cache || !v_cache || !out) return FCA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !(scale < INFINITY)) return FCA_ERR_INVALID_ARG;
    DeviceGuard dg(plan->device);
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return FCA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CUtensorMap tk, tv;
    if (!make_cache_map(&tk, k_cache, plan->num_blocks, plan->Hkv, plan->D) ||
        !make_cache_map(&tv, v_cache, plan->num_blocks, plan->Hkv, plan->D))
        return FCA_ERR_CUDA;
    const bool grouped = !plan->flat && plan->hdr.n_prefix_items > 0;
    const bool own = plan->async_update ? plan->cap_suffix_items > 0 : plan->hdr.n_suffix_items > 0;
    if (grouped) {
        // The two passes are independent.  With both, they share the SMs: the
        // grouped pass on its share, the per-request pass on the rest and then
        // on every SM the grouped pass leaves (programmatic serialization: it
        // starts once the grouped pass's CTAs all run, and ends after it).
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int np = own ? prefix_share(plan, sms) : 0;
        if (note_cuda(launch_prefix(plan, q, tk, tv, scale, np, s)) != cudaSuccess) return FCA_ERR_CUDA;
    }
    if (own && note_cuda(launch_suffix(plan, q, tk, tv, scale, grouped, s)) != cudaSuccess) return FCA_ERR_CUDA;
    // behind the per-request pass, which ends after the grouped one
    if (note_cuda(launch_merge(plan, out, lse, own, s)) != cudaSuccess) return FCA_ERR_CUDA;
    return FCA_OK;
}

fca_status fca_decode(const void* q, const void* k_cache, const void* v_cache, fca_plan_t plan, void* out,
                      float* lse, float scale, void* stream) {
    return decode_impl(q, k_cache, v_cache, plan, out, lse, scale, stream);
}

static fca_status pass_impl(int pass, const void* q, const void* k_cache, const void* v_cache, fca_plan_t plan,
                            float scale, void* stream) {
    if (!plan || !q || !k_cache || !v_cache) return FCA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !(scale < INFINITY)) return FCA_ERR_INVALID_ARG;
    DeviceGuard dg(plan->device);
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return FCA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CUtensorMap tk, tv;
    if (!make_cache_map(&tk, k_cache, plan->num_blocks, plan->Hkv, plan->D) ||
        !make_cache_map(&tv, v_cache, plan->num_blocks, plan->Hkv, plan->D))
        return FCA_ERR_CUDA;
    if (pass == 0) {
        if (plan->flat || plan->hdr.n_prefix_items == 0) return FCA_OK;
        return note_cuda(launch_prefix(plan, q, tk, tv, scale, 0, s)) == cudaSuccess ? FCA_OK
                                                                                                   : FCA_ERR_CUDA;
    }
    return note_cuda(launch_suffix(plan, q, tk, tv, scale, false, s)) == cudaSuccess ? FCA_OK : FCA_ERR_CUDA;
}

fca_status fca_prefix_pass(const void* q, const void* k_cache, const void* v_cache, fca_plan_t plan, float scale,
                           void* stream) {
    return pass_impl(0, q, k_cache, v_cache, plan, scale, stream);
}

fca_status fca_suffix_pass(const void* q, const void* k_cache, const void* v_cache, fca_plan_t plan, float scale,
                           void* stream) {
    return pass_impl(1, q, k_cache, v_cache, plan, scale, stream);
}

fca_status fca_merge_pass(fca_plan_t plan, void* out, float* lse, void* stream) {
    if (!plan || !out || !aligned16(out) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return FCA_ERR_INVALID_ARG;
    DeviceGuard dg(plan->device);
    return note_cuda(launch_merge(plan, out, lse, false, static_cast<cudaStream_t>(stream))) == cudaSuccess
               ? FCA_OK
               : FCA_ERR_CUDA;
}

fca_status fca_flat_decode(const void* q, const void* k_cache, const void* v_cache, fca_plan_t plan, void* out,
                           float* lse, float scale, void* stream) {
    if (!plan || !plan->flat) return FCA_ERR_INVALID_ARG;
    return decode_impl(q, k_cache, v_cache, plan, out, lse, scale, stream);
}

fca_status fca_plan_get_stats(fca_plan_t plan, fca_plan_stats* st) {
    if (!plan || !st) return FCA_ERR_INVALID_ARG;
    const PlanHeader& H = plan->hdr;
    const int64_t tok_bytes = (int64_t)plan->Hkv * plan->D * 2 * 2;
    st->num_requests = plan->R;
    st->num_groups = H.n_groups;
    st->max_depth = H.max_depth;
    st->num_q_heads = plan->Hq;
    st->num_kv_heads = plan->Hkv;
    st->head_dim = plan->D;
    st->split_tokens = H.split_tokens;
    st->prefix_split_tokens = H.prefix_split_tokens;
    st->prefix_items = H.n_prefix_items;
    st->suffix_items = H.n_suffix_items;
    st->num_partials = (int64_t)H.n_prefix_partials + H.n_suffix_partials;
    st->unique_kv_tokens = H.unique_kv_tokens;
    st->unique_kv_bytes = H.unique_kv_tokens * tok_bytes;
    st->flat_kv_bytes = H.flat_kv_tokens * tok_bytes;
    st->fca_kv_bytes = H.fca_kv_tokens * tok_bytes;
    st->prefix_kv_bytes = H.prefix_tok_sum * tok_bytes;
    st->suffix_kv_bytes = H.suffix_tok_sum * tok_bytes;
    st->workspace_bytes = (int64_t)plan->workspace_bytes;
    return FCA_OK;
}

fca_status fca_plan_member_count(fca_plan_t plan, int64_t* count) {
    if (!plan || !count) return FCA_ERR_INVALID_ARG;
    *count = plan->hdr.n_member_entries;
    return FCA_OK;
}

fca_status fca_plan_export(fca_plan_t plan, int32_t* a, int32_t* b, int32_t* parent, int32_t* member_off,
                           int32_t* n_members, int32_t* members, int32_t* suffix_start) {
    if (!plan) return FCA_ERR_INVALID_ARG;
    DeviceGuard dg(plan->device);
    if (cudaDeviceSynchronize() != cudaSuccess) {
        (void)cudaGetLastError();
        return FCA_ERR_CUDA;
    }
    const size_t ng = (size_t)plan->hdr.n_groups;
    struct Copy {
        int32_t* dst;
        const int32_t* src;
        size_t n;
    } copies[] = {{a, plan->g_a, ng},
                  {b, plan->g_b, ng},
                  {parent, plan->g_parent, ng},
                  {member_off, plan->g_moff, ng},
                  {n_members, plan->g_nm, ng},
                  {members, plan->members, (size_t)plan->hdr.n_member_entries},
                  {suffix_start, plan->suffix_start, (size_t)plan->R}};
    for (const Copy& c : copies) {
        if (!c.dst || c.n == 0) continue;
        if (cudaMemcpy(c.dst, c.src, c.n * sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess) {
            (void)cudaGetLastError();
            return FCA_ERR_CUDA;
        }
    }
    return FCA_OK;
}

fca_status fca_check_device_status(fca_plan_t plan, void* stream, int32_t* code) {
    if (!plan) return FCA_ERR_INVALID_ARG;
    DeviceGuard dg(plan->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess ||
        cudaMemcpy(&v, plan->dev_status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(plan->dev_status, 0, sizeof(v)) != cudaSuccess) {
        (void)cudaGetLastError();
        return FCA_ERR_CUDA;
    }
    if (code) *code = v;
    return v ? FCA_ERR_DEVICE_FLAG : FCA_OK;
}

const char* fca_status_string(fca_status status) {
    switch (status) {
        case FCA_OK: return "ok";
        case FCA_ERR_INVALID_ARG: return "invalid argument";
        case FCA_ERR_BAD_BLOCK_ID: return "block id out of range";
        case FCA_ERR_UNSUPPORTED: return "unsupported configuration";
        case FCA_ERR_CUDA: return "CUDA error";
        case FCA_ERR_OOM: return "out of device memory";
        case FCA_ERR_DEVICE_FLAG: return "kernel reported an internal error";
        case FCA_ERR_TOO_LARGE: return "problem larger than the fixed scratch of fca_paged_decode_static";
    }
    return "unknown status";
}

const char* fca_version(void) { return "fca_b200 0.1.0 sm_100a"; }

const char* fca_last_cuda_error(void) { return cudaGetErrorString(g_last_error); }

}  // extern "C"
