// Dense attention forward on sm_100a (the LazyFlash forward is FlashAttention's,
// unchanged: article standfirst and section "Le passage arrière fait deux fois
// le travail du passage avant").
//
// One CTA computes a 128-row query tile of one head of one segment:
//   TMA:      Q tile once, K/V tiles double-buffered (128 x d, SW128 panels);
//   tcgen05:  S = Q K^T into TMEM (128 lanes x 128 fp32 columns),
//             O += P V into TMEM (128 lanes x d columns);
//   4 warps:  thread r owns query row r (TMEM lane r): online softmax in the
//             exp2 domain, P rounded to bf16 into shared memory in the
//             tensor core's K-major layout, O rescaled in TMEM when the row
//             maximum moves;
//   epilogue: O / l -> bf16, LSE = ln(l) + max (natural log).
#pragma once

#include "lf_device.cuh"

namespace lf {

struct FwdParams {
    const int32_t* cu_seqlens;
    int T, hq, hkv, causal, max_seqlen;
    float scale_log2;          // softmax_scale * log2(e)
    __nv_bfloat16* o;
    float* lse;
};

template <int D>
struct FwdSmem {
    static constexpr int kPanels = D / 64;
    static constexpr uint32_t kTile = kPanels * kPanelBytes;     // one 128 x D bf16 tile
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kTile;                   // 2 stages
    static constexpr uint32_t kV = kK + 2 * kTile;               // 2 stages
    static constexpr uint32_t kP = kV + 2 * kTile;               // 128 x 128 bf16
    static constexpr uint32_t kBars = kP + 2 * kPanelBytes;
    static constexpr uint32_t kBytes = kBars + 64;
    static constexpr uint32_t kAlloc = kBytes + 1024;            // slack for 1024-B alignment
};

constexpr int kFwdThreads = 128;

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, FwdParams prm) {
    using L = FwdSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar_q = reinterpret_cast<uint64_t*>(smem + L::kBars);
    uint64_t* bar_kv = bar_q + 1;     // [2]
    uint64_t* bar_mma = bar_q + 3;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_q + 4);
    int* abort_flag = reinterpret_cast<int*>(bar_q + 5);

    const int h = blockIdx.x;
    const int s = blockIdx.z;
    int seg0, len;
    if (!load_segment(prm.cu_seqlens, s, prm.T, prm.max_seqlen, seg0, len, 20)) return;
    const int ntiles = (len + 127) >> 7;
    const int qt = ntiles - 1 - static_cast<int>(blockIdx.y);   // longest rows first
    if (qt < 0) return;
    const int g = h / (prm.hq / prm.hkv);
    const int nkv = prm.causal ? qt + 1 : ntiles;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t s_base = smem_addr(smem);

    if (tid == 0) {
        mbar_init(bar_q, 1);
        mbar_init(&bar_kv[0], 1);
        mbar_init(&bar_kv[1], 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_s = tmem;            // S: columns [0, 128)
    const uint32_t t_o = tmem + 128;      // O: columns [128, 128 + D)
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;

    const int row0 = seg0 + qt * 128;
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_q, L::kTile);
        for (int c = 0; c < L::kPanels; ++c)
            tma_load_3d(smem + L::kQ + c * kPanelBytes, &tm_q, bar_q, c * 64, h, row0);
        mbar_arrive_expect_tx(&bar_kv[0], 2 * L::kTile);
        for (int c = 0; c < L::kPanels; ++c) {
            tma_load_3d(smem + L::kK + c * kPanelBytes, &tm_k, &bar_kv[0], c * 64, g, seg0);
            tma_load_3d(smem + L::kV + c * kPanelBytes, &tm_v, &bar_kv[0], c * 64, g, seg0);
        }
    }

    constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t kIdescO = idesc_bf16(128, D, 0, 1);
    const int q_local = qt * 128 + tid;     // this thread's query row within the segment
    float m_run = -INFINITY, l_run = 0.f;
    uint32_t mma_phase = 0;
    bool ok = true;
    // loads issued / waited per K-V stage (thread 0 only), for the drain on abort
    int kv_issued[2] = {1, 0}, kv_waited[2] = {0, 0};
    bool q_waited = false;

    for (int j = 0; j < nkv && ok; ++j) {
        const int st = j & 1;
        if (tid == 0) {
            if (j + 1 < nkv) {
                const int ns = st ^ 1;
                mbar_arrive_expect_tx(&bar_kv[ns], 2 * L::kTile);
                ++kv_issued[ns];
                for (int c = 0; c < L::kPanels; ++c) {
                    tma_load_3d(smem + L::kK + ns * L::kTile + c * kPanelBytes, &tm_k, &bar_kv[ns],
                                c * 64, g, seg0 + (j + 1) * 128);
                    tma_load_3d(smem + L::kV + ns * L::kTile + c * kPanelBytes, &tm_v, &bar_kv[ns],
                                c * 64, g, seg0 + (j + 1) * 128);
                }
            }
            bool w_ok = q_waited || mbar_wait(bar_q, 0, 1);
            q_waited = w_ok;
            w_ok = w_ok && mbar_wait(&bar_kv[st], (j >> 1) & 1, 2);
            if (w_ok) ++kv_waited[st];
            if (w_ok) {
                tc_fence_after();
                const uint32_t qa = s_base + L::kQ;
                const uint32_t ka = s_base + L::kK + st * L::kTile;
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    mma_bf16_ss(t_s, desc_kmajor(qa, k), desc_kmajor(ka, k), kIdescS, k > 0);
                mma_commit(bar_mma);
            } else {
                *abort_flag = 1;
            }
        }
        __syncthreads();
        if (*abort_flag) { ok = false; break; }
        if (!mbar_wait(bar_mma, mma_phase, 3)) *abort_flag = 1;
        mma_phase ^= 1;
        __syncthreads();
        if (*abort_flag) { ok = false; break; }
        tc_fence_after();

        // ---- online softmax on this thread's row ----
        float sv[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float tmp[32];
            tmem_ld32(t_s + lane_off + c * 32, tmp);
#pragma unroll
            for (int e = 0; e < 32; ++e) sv[c * 32 + e] = tmp[e];
        }
        const int kv0 = j * 128;
        const bool diag = prm.causal ? (kv0 + 127 > q_local) : false;
        const bool tail = kv0 + 128 > len;
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 128; ++e) {
            const int kv = kv0 + e;
            const bool valid = !(diag && kv > q_local) && !(tail && kv >= len);
            sv[e] = valid ? sv[e] * prm.scale_log2 : -INFINITY;
            mx = fmaxf(mx, sv[e]);
        }
        const float m_new = fmaxf(m_run, mx);
        const float alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
        float rs = 0.f;
        const uint32_t p_base = s_base + L::kP;
#pragma unroll
        for (int ch = 0; ch < 16; ++ch) {
            uint32_t pk[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                const float p0 = fast_exp2(sv[ch * 8 + 2 * e2] - m_new);
                const float p1 = fast_exp2(sv[ch * 8 + 2 * e2 + 1] - m_new);
                rs += p0 + p1;
                pk[e2] = pack_bf16(p0, p1);
            }
            st_shared_v4(p_base + sw128_chunk_offset(tid, ch), pk[0], pk[1], pk[2], pk[3]);
        }
        l_run = l_run * alpha + rs;
        m_run = m_new;
        // rescale the running O when this row's maximum moved
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                float ov[32];
                tmem_ld32(t_o + lane_off + c * 32, ov);
#pragma unroll
                for (int e = 0; e < 32; ++e) ov[e] *= alpha;
                tmem_st32(t_o + lane_off + c * 32, ov);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t va = s_base + L::kV + st * L::kTile;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16_ss(t_o, desc_kmajor(p_base, k), desc_mnmajor(va, k), kIdescO,
                            (j > 0 || k > 0) ? 1u : 0u);
            mma_commit(bar_mma);
        }
        if (!mbar_wait(bar_mma, mma_phase, 4)) *abort_flag = 1;
        mma_phase ^= 1;
        __syncthreads();
        if (*abort_flag) { ok = false; break; }
        tc_fence_after();
    }

    if (ok) {
        // ---- epilogue: O / l -> bf16, LSE ----
        const bool row_ok = q_local < len;
        const float inv_l = 1.f / l_run;
        const int t = seg0 + q_local;
        __nv_bfloat16* orow = prm.o + ((size_t)t * prm.hq + h) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            float ov[32];
            tmem_ld32(t_o + lane_off + c * 32, ov);
            if (row_ok) {
#pragma unroll
                for (int e8 = 0; e8 < 4; ++e8) {
                    uint4 pk;
                    pk.x = pack_bf16(ov[e8 * 8 + 0] * inv_l, ov[e8 * 8 + 1] * inv_l);
                    pk.y = pack_bf16(ov[e8 * 8 + 2] * inv_l, ov[e8 * 8 + 3] * inv_l);
                    pk.z = pack_bf16(ov[e8 * 8 + 4] * inv_l, ov[e8 * 8 + 5] * inv_l);
                    pk.w = pack_bf16(ov[e8 * 8 + 6] * inv_l, ov[e8 * 8 + 7] * inv_l);
                    *reinterpret_cast<uint4*>(orow + c * 32 + e8 * 8) = pk;
                }
            }
        }
        if (row_ok)
            prm.lse[(size_t)h * prm.T + t] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
    }
    if (!ok && tid == 0) {
        // a wait gave up: let this CTA's own TMA copies land (bounded) before exit
        if (!q_waited) mbar_wait(bar_q, 0, 5);
        for (int st = 0; st < 2; ++st)
            while (kv_waited[st] < kv_issued[st] && mbar_wait(&bar_kv[st], kv_waited[st] & 1, 5))
                ++kv_waited[st];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace lf
