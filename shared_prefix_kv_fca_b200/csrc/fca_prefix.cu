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
// One CTA per work item = (group, KV head, 128-row Q tile, token chunk); 192
// threads in three roles:
//   warp 0      TMA producer: streams 64-token stages of K and V (four paged
//               16-token blocks, two 64-column halves each, 128-byte swizzle)
//               into a ring of kPreStages slots; blocks past the chunk are
//               loaded from out-of-range rows, i.e. as zeros;
//   warp 1      allocates tensor memory and, from one thread, issues
//               S = Q K^T (M=128, N=64, K=head_dim) into one of two S buffers
//               and O_s = P V (M=128, N=head_dim, K=64) into one of two O
//               buffers, signalling completions with tcgen05.commit;
//   warps 2-5   softmax: thread = query row (TMEM lane); read the S row,
//               online max / sum in fp32 (log2 domain), write P as bf16 into
//               shared memory in the MMA's K-major swizzled layout, then fold
//               the previous stage's O_s into a register accumulator with the
//               running rescale factor.
// The S buffer of stage j+1 is computed while stage j's softmax runs.
// Output: one partial row (normalised o, natural-log lse) per stacked query
// row, merged later with the row's other partials.
#include <cuda_bf16.h>

#include "fca_device.cuh"
#include "fca_internal.h"

namespace fca {

namespace {

constexpr int kPreStages = 4;
constexpr int kPreThreads = 192;

struct PrefixArgs {
    const PrefixItem* items;
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
    static constexpr int kQ = kHalves * 128 * 128;        // Q tile, bytes
    static constexpr int kKV = kHalves * 64 * 128;        // one 64-token K (or V) stage
    static constexpr int kP = 128 * 128;                  // one P buffer (128 rows x 64 bf16)
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQ;
    static constexpr int kOffV = kOffK + kPreStages * kKV;
    static constexpr int kOffP = kOffV + kPreStages * kKV;
    static constexpr int kOffBar = kOffP + 2 * kP;
    // barriers: q_full, k_full[S], v_full[S], kv_empty[S], s_full[2], s_free[2],
    //           p_full[2], o_full[2], o_free[2], mma_done
    static constexpr int kNumBars = 1 + 3 * kPreStages + 10 + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kTotal = kOffMisc + 64 + 1024;   // + alignment slack
    static constexpr uint32_t kTmemCols = D == 128 ? 512 : 256;
    static constexpr uint32_t kColS = 0;                  // two 64-column S buffers
    static constexpr uint32_t kColO = 128;                // two D-column O buffers
};

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
    uint64_t* kv_empty = v_full + kPreStages;
    uint64_t* s_full = kv_empty + kPreStages;
    uint64_t* s_free = s_full + 2;
    uint64_t* p_full = s_free + 2;
    uint64_t* o_full = p_full + 2;
    uint64_t* o_free = o_full + 2;
    uint64_t* mma_done = o_free + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 16);

    const PrefixItem it = a.items[blockIdx.x];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t n_tok = it.tok1 - it.tok0;
    const int32_t n_stages = (n_tok + kStageTokens - 1) / kStageTokens;

    if (threadIdx.x == 0) {
        dev::mbar_init(q_full, 128);
        for (int s = 0; s < kPreStages; ++s) {
            dev::mbar_init(&k_full[s], 1);
            dev::mbar_init(&v_full[s], 1);
            dev::mbar_init(&kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            dev::mbar_init(&s_full[b], 1);
            dev::mbar_init(&s_free[b], 128);
            dev::mbar_init(&p_full[b], 128);
            dev::mbar_init(&o_full[b], 1);
            dev::mbar_init(&o_free[b], 128);
        }
        dev::mbar_init(mma_done, 1);
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
        if (lane == 0) {
            dev::tma_prefetch_desc(&tmK);
            dev::tma_prefetch_desc(&tmV);
            const int32_t* row = a.bt + (int64_t)it.bt_row * a.max_blocks;
            const int32_t blk0 = it.tok0 / kBlockSize, blk_end = it.tok1 / kBlockSize;
            int32_t issued = 0;
            for (int32_t j = 0; j < n_stages; ++j) {
                const int s = j % kPreStages;
                if (j >= kPreStages &&
                    !dev::mbar_wait(&kv_empty[s], ((j / kPreStages) - 1) & 1, abort_flag, a.err))
                    break;
                uint8_t* kdst = smem + L::kOffK + s * L::kKV;
                uint8_t* vdst = smem + L::kOffV + s * L::kKV;
                dev::mbar_arrive_expect_tx(&k_full[s], L::kKV);
                dev::mbar_arrive_expect_tx(&v_full[s], L::kKV);
#pragma unroll
                for (int bi = 0; bi < kStageTokens / kBlockSize; ++bi) {
                    const int32_t blk = blk0 + j * (kStageTokens / kBlockSize) + bi;
                    // past the chunk: rows beyond the cache, which TMA fills with zeros
                    const int32_t trow = blk < blk_end ? row[blk] * kBlockSize : a.num_blocks * kBlockSize;
#pragma unroll
                    for (int hf = 0; hf < L::kHalves; ++hf) {
                        dev::tma_load_3d(kdst + hf * (64 * 128) + bi * 2048, &tmK, &k_full[s], hf * 64, it.head,
                                         trow);
                        dev::tma_load_3d(vdst + hf * (64 * 128) + bi * 2048, &tmV, &v_full[s], hf * 64, it.head,
                                         trow);
                    }
                }
                ++issued;
            }
            for (int32_t j = issued - 1; j >= 0 && j >= issued - kPreStages; --j) {
                volatile int never = 0;
                dev::mbar_wait(&k_full[j % kPreStages], (j / kPreStages) & 1, &never, a.err);
                dev::mbar_wait(&v_full[j % kPreStages], (j / kPreStages) & 1, &never, a.err);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = dev::idesc_bf16_f32(128, 64, false, false);
            constexpr uint32_t idesc_pv = dev::idesc_bf16_f32(128, D, false, true);
            const uint32_t q_base = dev::smem_u32(smem + L::kOffQ);
            bool ok = dev::mbar_wait(q_full, 0, abort_flag, a.err);
            auto issue_qk = [&](int32_t j) -> bool {
                const int s = j % kPreStages, sb = j & 1;
                if (!dev::mbar_wait(&k_full[s], (j / kPreStages) & 1, abort_flag, a.err)) return false;
                if (j >= 2 && !dev::mbar_wait(&s_free[sb], ((j >> 1) - 1) & 1, abort_flag, a.err)) return false;
                dev::tc_fence_after();
                const uint32_t k_base = dev::smem_u32(smem + L::kOffK + s * L::kKV);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint64_t ad = dev::smem_desc_sw128(q_base + (k >> 2) * (128 * 128) + (k & 3) * 32, 16, 1024);
                    const uint64_t bd = dev::smem_desc_sw128(k_base + (k >> 2) * (64 * 128) + (k & 3) * 32, 16, 1024);
                    dev::tc_mma_ss(tmem + L::kColS + sb * 64, ad, bd, idesc_qk, k > 0 ? 1u : 0u);
                }
                dev::tc_commit(&s_full[sb]);
                return true;
            };
            if (ok && n_stages > 0) ok = issue_qk(0);
            for (int32_t j = 0; ok && j < n_stages; ++j) {
                if (j + 1 < n_stages && !issue_qk(j + 1)) { ok = false; break; }
                const int s = j % kPreStages, pb = j & 1;
                if (!dev::mbar_wait(&p_full[pb], (j >> 1) & 1, abort_flag, a.err)) { ok = false; break; }
                if (j >= 2 && !dev::mbar_wait(&o_free[pb], ((j >> 1) - 1) & 1, abort_flag, a.err)) { ok = false; break; }
                if (!dev::mbar_wait(&v_full[s], (j / kPreStages) & 1, abort_flag, a.err)) { ok = false; break; }
                dev::tc_fence_after();
                const uint32_t p_base = dev::smem_u32(smem + L::kOffP + pb * L::kP);
                const uint32_t v_base = dev::smem_u32(smem + L::kOffV + s * L::kKV);
#pragma unroll
                for (int k = 0; k < kStageTokens / 16; ++k) {
                    const uint64_t ad = dev::smem_desc_sw128(p_base + k * 32, 16, 1024);
                    const uint64_t bd = dev::smem_desc_sw128(v_base + k * 2048, 64 * 128, 1024);
                    dev::tc_mma_ss(tmem + L::kColO + pb * D, ad, bd, idesc_pv, k > 0 ? 1u : 0u);
                }
                dev::tc_commit(&o_full[pb]);
                dev::tc_commit(&kv_empty[s]);
            }
            // every MMA of this thread has retired before tensor memory is freed
            dev::tc_commit(mma_done);
            volatile int never = 0;
            dev::mbar_wait(mma_done, 0, &never, a.err);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax warps
        const int quarter = warp & 3;                 // TMEM lane quarter this warp may access
        const int r = quarter * 32 + lane;            // tile row
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const bool row_valid = r < it.nrows;

        // Q tile row r: stacked row it.row0 + r = member (i / G), query head (head * G + i % G)
        {
            uint8_t* qdst = smem + L::kOffQ;
            const __nv_bfloat16* src = nullptr;
            if (row_valid) {
                const int32_t i = it.row0 + r;
                const int32_t member = a.members[a.g_moff[it.group] + i / a.G];
                src = a.q + ((int64_t)member * a.Hq + it.head * a.G + i % a.G) * D;
            }
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                uint4 v = make_uint4(0, 0, 0, 0);
                if (row_valid) v = *reinterpret_cast<const uint4*>(src + c * 8);
                const int hf = c >> 3, cc = c & 7;
                *reinterpret_cast<uint4*>(qdst + hf * (128 * 128) + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
            }
            dev::fence_proxy_async_smem();
            dev::mbar_arrive(q_full);
        }

        float m_run = -INFINITY, l_run = 0.f, alpha_last = 0.f;
        float oacc[D];
#pragma unroll
        for (int d = 0; d < D; ++d) oacc[d] = 0.f;
        bool ok = true;

        auto fold = [&](int32_t jj, float al) -> bool {
            const int ob = jj & 1;
            const bool got = dev::mbar_wait(&o_full[ob], (jj >> 1) & 1, abort_flag, a.err);
            if (!__all_sync(0xffffffffu, got)) return false;     // tcgen05.ld needs the whole warp
            dev::tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                dev::tmem_ld32(tmem + lane_base + L::kColO + ob * D + c * 32, v);
                dev::tc_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) oacc[c * 32 + i] = fmaf(oacc[c * 32 + i], al, __uint_as_float(v[i]));
            }
            dev::tc_fence_before();
            dev::mbar_arrive(&o_free[ob]);
            return true;
        };

        for (int32_t j = 0; j < n_stages; ++j) {
            const int sb = j & 1;
            const bool got = dev::mbar_wait(&s_full[sb], (j >> 1) & 1, abort_flag, a.err);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            dev::tc_fence_after();
            uint32_t s_lo[32], s_hi[32];
            dev::tmem_ld32(tmem + lane_base + L::kColS + sb * 64, s_lo);
            dev::tmem_ld32(tmem + lane_base + L::kColS + sb * 64 + 32, s_hi);
            dev::tc_wait_ld();
            dev::tc_fence_before();
            dev::mbar_arrive(&s_free[sb]);

            const int32_t n_valid = min(kStageTokens, n_tok - j * kStageTokens);
            float sv[64];
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float raw = __uint_as_float(i < 32 ? s_lo[i & 31] : s_hi[i & 31]);
                const float x = i < n_valid ? raw * a.scale_log2 : -INFINITY;
                sv[i] = x;
                mx = fmaxf(mx, x);
            }
            const float m_new = fmaxf(m_run, mx);
            const float alpha = exp2f(m_run - m_new);
            float psum = 0.f;
            uint8_t* prow = smem + L::kOffP + sb * L::kP + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    p[e] = exp2f(sv[c * 8 + e] - m_new);
                    psum += p[e];
                }
                uint4 packed;
                packed.x = dev::pack_bf16x2(p[0], p[1]);
                packed.y = dev::pack_bf16x2(p[2], p[3]);
                packed.z = dev::pack_bf16x2(p[4], p[5]);
                packed.w = dev::pack_bf16x2(p[6], p[7]);
                *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = packed;
            }
            l_run = l_run * alpha + psum;
            m_run = m_new;
            dev::fence_proxy_async_smem();
            dev::mbar_arrive(&p_full[sb]);
            if (j > 0 && !fold(j - 1, alpha_last)) { ok = false; break; }
            alpha_last = alpha;
        }
        if (ok && n_stages > 0) ok = fold(n_stages - 1, alpha_last);

        if (ok && row_valid) {
            const float inv = 1.f / l_run;
            float* dst = a.part_o + ((int64_t)it.part_row0 + r) * D;
#pragma unroll
            for (int d = 0; d < D; d += 4)
                *reinterpret_cast<float4*>(dst + d) =
                    make_float4(oacc[d] * inv, oacc[d + 1] * inv, oacc[d + 2] * inv, oacc[d + 3] * inv);
            a.part_lse[it.part_row0 + r] = (m_run + log2f(l_run)) * 0.69314718055994531f;
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
cudaError_t launch_prefix_t(const PrefixArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, int n_items,
                            cudaStream_t stream) {
    using L = PreLayout<D>;
    cudaError_t e = cudaFuncSetAttribute(k_prefix<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal);
    if (e != cudaSuccess) return e;
    k_prefix<D><<<n_items, kPreThreads, L::kTotal, stream>>>(a, tk, tv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefix(const fca_plan_s* P, const void* q, const CUtensorMap& tk, const CUtensorMap& tv,
                          float scale, cudaStream_t stream) {
    const int n = P->hdr.n_prefix_items;
    if (n == 0) return cudaSuccess;
    PrefixArgs a;
    a.items = P->prefix_items;
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
    if (P->D == 128) return launch_prefix_t<128>(a, tk, tv, n, stream);
    return launch_prefix_t<64>(a, tk, tv, n, stream);
}

}  // namespace fca
