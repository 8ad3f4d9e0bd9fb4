// Dense attention forward on sm_100a (the LazyFlash forward is FlashAttention's,
// unchanged: article standfirst and section "Le passage arrière fait deux fois
// le travail du passage avant").
//
// One CTA computes two consecutive 128-row query tiles (2m, 2m+1) of one head
// of one segment, in ping-pong: while one softmax warpgroup turns its score
// tile into probabilities, the tensor core computes the other tile's scores
// and P.V products.
//   TMA:      both Q tiles once; K and V tiles through two-stage rings;
//   tcgen05:  S_t = Q_t K_j^T (SS, 128 x 128 fp32 in TMEM), O_t += P_t V_j
//             (TS: P_t read from TMEM, where the softmax wrote it over S_t);
//   softmax:  warpgroup t, thread r owns query row r (TMEM lane r): online
//             softmax in the exp2 domain with a stale-max rule (the reference
//             maximum moves only when the row maximum grows by more than 2^8,
//             and only then is O rescaled in TMEM); P is written in four
//             32-column chunks, and P.V starts once the first half is stored;
//   epilogue: O / l -> bf16, LSE = (m + log2 l) * ln 2.
// Roles (384 threads): warp 0 TMA producer, warps 1 and 2 MMA issuers of tile 0
// and tile 1 (whole warp, one elected lane issues; the two take turns so the
// tensor pipe sees the ping-pong order), warps 4-7 softmax of tile 0, warps
// 8-11 softmax of tile 1.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d),
// O1 [384,384+d); P_t (bf16, packed two per column) over S_t [0,64).  Reuse
// of a region by a later MMA relies on tcgen05.mma executing in issue order.
#pragma once

#include <climits>

#include "lf_device.cuh"

namespace lf {

struct FwdParams {
    const int32_t* cu_seqlens;
    int T, hq, hkv, causal, max_seqlen, nseq;
    float scale_log2;          // softmax_scale * log2(e)
    int tile_major;            // CTA order: 1 = KV head fastest (see the kernel)
    __nv_bfloat16* o;
    float* lse;
};

template <int D>
struct FwdSmem {
    static constexpr int kPanels = D / 64;
    static constexpr uint32_t kTile = kPanels * kPanelBytes;     // one 128 x D bf16 tile
    static constexpr uint32_t kQ = 0;                            // 2 tiles
    static constexpr uint32_t kK = kQ + 2 * kTile;               // 2 stages
    static constexpr uint32_t kV = kK + 2 * kTile;               // 2 stages
    static constexpr uint32_t kBars = kV + 2 * kTile;
    static constexpr uint32_t kBytes = kBars + 256;
    static constexpr uint32_t kAlloc = kBytes + 1024;            // slack for 1024-B alignment
};

constexpr int kFwdThreads = 384;
constexpr int kFwdLaunchRegs = 168;     // 65536 / 384, rounded down to a multiple of 8
constexpr int kFwdCtrlRegs = 64;
constexpr int kFwdSoftmaxRegs = 216;
constexpr float kRescaleThreshold = 8.0f;   // log2 of the largest P before a rescale

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, FwdParams prm) {
    using L = FwdSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
    uint64_t* bar_q = bars + 0;
    uint64_t* bar_k_full = bars + 1;    // [2]
    uint64_t* bar_k_empty = bars + 3;   // [2]
    uint64_t* bar_v_full = bars + 5;    // [2]
    uint64_t* bar_v_empty = bars + 7;   // [2]
    uint64_t* bar_s_full = bars + 9;    // [2] per query tile
    uint64_t* bar_p_ready = bars + 11;  // [2]
    uint64_t* bar_o_done = bars + 13;   // [2]
    uint64_t* bar_done = bars + 15;     // [2] per MMA issuer
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 18);
    volatile int* burst_seq = reinterpret_cast<volatile int*>(bars + 19);   // [2] bursts issued per MMA issuer
    uint64_t* bar_p_half = bars + 20;   // [2] per query tile: P columns [0, 64) written

    // blockIdx.x = pair * G + query head within the KV head's group, the pairs of
    // 256 query rows running over all segments, segment by segment; blockIdx.y = KV
    // head.  The G query heads that share a KV head run together, longest rows first
    // within each segment, so their K/V stay in L2 and each group's work outlasts its
    // heaviest CTA.  With few waves of CTAs (tile_major) the KV head runs fastest
    // instead, so that every KV head's longest rows start first rather than the last
    // head's running alone at the end.
    const int G = prm.hq / prm.hkv;
    int g, xr;
    if (prm.tile_major) {
        const int lin = static_cast<int>(blockIdx.x + blockIdx.y * gridDim.x);
        g = lin % static_cast<int>(gridDim.y);
        xr = lin / static_cast<int>(gridDim.y);
    } else {
        g = blockIdx.y;
        xr = blockIdx.x;
    }
    const int h = g * G + xr % G;
    const int pg = xr / G;
    const int s = segment_of_unit(prm.cu_seqlens, prm.nseq, pg, 8);
    if (s < 0) return;
    int seg0, len;
    if (!load_segment(prm.cu_seqlens, s, prm.T, prm.max_seqlen, seg0, len, 20)) return;
    const int ntiles = (len + 127) >> 7;
    const int npairs = (ntiles + 1) >> 1;
    const int m = npairs - 1 - (pg - first_unit_of_segment(seg0, s, 8));   // longest rows first
    if (m < 0) return;
    const bool two = 2 * m + 1 < ntiles;                     // tile 1 exists
    // KV tiles each query tile needs
    const int nkv0 = prm.causal ? 2 * m + 1 : ntiles;
    const int nkv1 = two ? (prm.causal ? 2 * m + 2 : ntiles) : 0;
    const int nkv = nkv0 > nkv1 ? nkv0 : nkv1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t s_base = smem_addr(smem);

    if (tid == 0) {
        mbar_init(bar_q, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_k_full[i], 1);
            mbar_init(&bar_k_empty[i], two ? 2 : 1);   // one commit per query tile
            mbar_init(&bar_v_full[i], 1);
            mbar_init(&bar_v_empty[i], two ? 2 : 1);
            mbar_init(&bar_s_full[i], 1);
            mbar_init(&bar_p_ready[i], 128);
            mbar_init(&bar_p_half[i], 128);
            mbar_init(&bar_o_done[i], 1);
        }
        mbar_init(&bar_done[0], 1);
        mbar_init(&bar_done[1], 1);
        *abort_flag = 0;
        burst_seq[0] = 0;
        burst_seq[1] = two ? 0 : INT_MAX;   // a lone tile never waits for its turn
        fence_barrier_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // 384 threads x 168 registers at launch >= 128 x 64 (TMA, MMA, idle) + 256 x 216 (softmax)
    static_assert(128 * kFwdCtrlRegs + 256 * kFwdSoftmaxRegs <= kFwdThreads * kFwdLaunchRegs, "register split");
    if (warp < 4) {
        regs_release_to<kFwdCtrlRegs>();
        if (warp == 0) {
            // ===================== TMA producer =====================
            if (lane == 0) {
                const uint32_t qbytes = (two ? 2 : 1) * L::kTile;
                mbar_arrive_expect_tx(bar_q, qbytes);
                for (int t = 0; t < (two ? 2 : 1); ++t)
                    for (int c = 0; c < L::kPanels; ++c)
                        tma_load_3d(smem + L::kQ + t * L::kTile + c * kPanelBytes, &tm_q, bar_q, c * 64, h,
                                    seg0 + (2 * m + t) * 128);
                uint32_t kpar[2] = {0, 0}, vpar[2] = {0, 0};
                int kfill = 0, vfill = 0;   // loads issued (for the drain on abort)
                for (int j = 0; j < nkv; ++j) {
                    const int st = j & 1;
                    if (j >= 2 && !mbar_wait_or_abort(&bar_k_empty[st], ((j >> 1) - 1) & 1, 21, abort_flag)) break;
                    mbar_arrive_expect_tx(&bar_k_full[st], L::kTile);
                    for (int c = 0; c < L::kPanels; ++c)
                        tma_load_3d(smem + L::kK + st * L::kTile + c * kPanelBytes, &tm_k, &bar_k_full[st],
                                    c * 64, g, seg0 + j * 128);
                    kpar[st] = (j >> 1) & 1;
                    ++kfill;
                    if (j >= 2 && !mbar_wait_or_abort(&bar_v_empty[st], ((j >> 1) - 1) & 1, 22, abort_flag)) break;
                    mbar_arrive_expect_tx(&bar_v_full[st], L::kTile);
                    for (int c = 0; c < L::kPanels; ++c)
                        tma_load_3d(smem + L::kV + st * L::kTile + c * kPanelBytes, &tm_v, &bar_v_full[st],
                                    c * 64, g, seg0 + j * 128);
                    vpar[st] = (j >> 1) & 1;
                    ++vfill;
                }
                if (*abort_flag) {
                    // let this CTA's own copies land before the CTA exits (bounded)
                    mbar_wait(bar_q, 0, 23);
                    for (int st = 0; st < 2; ++st) {
                        if (kfill > st) mbar_wait(&bar_k_full[st], kpar[st], 23);
                        if (vfill > st) mbar_wait(&bar_v_full[st], vpar[st], 23);
                    }
                }
            }
            __syncwarp();
        } else if (warp == 1 || warp == 2) {
            // ============ MMA issuers: warp 1 for query tile 0, warp 2 for tile 1 ============
            // The tensor pipe sees the bursts in the single-issuer order S0 S1 | PV0 S0' |
            // PV1 S1' | ..., so each tile's softmax overlaps the other tile's MMAs, but each
            // issuer clears its own barrier waits while the other one's burst runs.  A burst
            // waits for its turn on the other issuer's count of bursts issued.  The whole
            // warp runs this code (one elected lane issues); every wait result is made
            // warp-uniform.  Each commit tracks only the MMAs of the issuing lane.
            const int t = warp - 1;
            const int nk = t ? nkv1 : nkv0;
            if (nk > 0) {
                constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);
                constexpr uint32_t kIdescO = idesc_bf16(128, D, 0, 1);
                const uint32_t qa = s_base + L::kQ + t * L::kTile;
                const uint32_t t_s = tmem + t * 128, t_o = tmem + 256 + t * 128;
                int nb = 0;   // bursts this warp has issued
                auto wait = [&](uint64_t* bar, uint32_t parity, int site) {
                    return __all_sync(0xffffffffu, mbar_wait_or_abort(bar, parity, site, abort_flag));
                };
                auto my_turn = [&]() {
                    return __all_sync(0xffffffffu, spin_until_geq(&burst_seq[1 - t], nb + t, 19, abort_flag));
                };
                auto publish = [&](int v) {
                    __syncwarp();
                    if (lane == 0) burst_seq[t] = v;
                    __syncwarp();
                };
                auto issue_s = [&](int j) {
                    const uint32_t ka = s_base + L::kK + (j & 1) * L::kTile;
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        mma_bf16_ss_warp(t_s, desc_kmajor(qa, k), desc_kmajor(ka, k), kIdescS, k > 0);
                    mma_commit_warp(&bar_s_full[t]);
                    mma_commit_warp(&bar_k_empty[j & 1]);
                };
                bool ok = wait(bar_q, 0, 24) && wait(&bar_k_full[0], 0, 25) && my_turn();
                if (ok) {
                    tc_fence_after();
                    issue_s(0);
                    publish(++nb);
                }
                for (int j = 0; j < nk && ok; ++j) {
                    const int st = j & 1;
                    if (!wait(&bar_v_full[st], (j >> 1) & 1, 26)) break;
                    if (j + 1 < nk && !wait(&bar_k_full[(j + 1) & 1], ((j + 1) >> 1) & 1, 28)) break;
                    if (!wait(&bar_p_half[t], j & 1, 18)) break;
                    if (!my_turn()) break;
                    // P.V over the first 64 keys while the softmax finishes the second half
                    tc_fence_after();
                    const uint32_t va = s_base + L::kV + st * L::kTile;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16_ts_warp(t_o, t_s + k * 8, desc_mnmajor(va, k), kIdescO, (j > 0 || k > 0) ? 1u : 0u);
                    if (!wait(&bar_p_ready[t], j & 1, 27)) break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 4; k < 8; ++k)
                        mma_bf16_ts_warp(t_o, t_s + k * 8, desc_mnmajor(va, k), kIdescO, 1u);
                    mma_commit_warp(&bar_o_done[t]);
                    mma_commit_warp(&bar_v_empty[st]);
                    if (j + 1 < nk) issue_s(j + 1);
                    publish(++nb);
                }
                publish(INT_MAX);   // finished (or aborted): never hold the other issuer
                mma_commit_warp(&bar_done[t]);
                // every MMA issued by this warp has finished (waits even after an abort)
                __all_sync(0xffffffffu, mbar_wait(&bar_done[t], 0, 29));
            }
        }
    } else {
        regs_grow_to<kFwdSoftmaxRegs>();
        // ============ softmax, one warpgroup per query tile (thread = row) ============
        const int t = (warp - 4) >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + t * 128 + lane_off;
        const uint32_t t_o = tmem + 256 + t * 128 + lane_off;
        const int nk = t ? nkv1 : nkv0;
        const int qt = 2 * m + t;
        const int q_local = qt * 128 + r;
        float m_ref = -INFINITY, l_run = 0.f;
        bool failed = false;
        for (int j = 0; j < nk; ++j) {
            const bool got = mbar_wait_or_abort(&bar_s_full[t], j & 1, 30, abort_flag);
            if (!__all_sync(0xffffffffu, got)) { failed = true; break; }
            tc_fence_after();
            // the row's 128 score columns: eight loads in flight, one wait
            float sv[128];
            {
                uint32_t sr[8][16];
#pragma unroll
                for (int c = 0; c < 8; ++c) tmem_ld16_nowait(t_s + c * 16, sr[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    tmem_regs_ready(sr[c]);
#pragma unroll
                    for (int e = 0; e < 16; ++e) sv[c * 16 + e] = __uint_as_float(sr[c][e]);
                }
            }
            const int kv0 = j * 128;
            const bool diag = prm.causal && j == qt;
            const bool tail = kv0 + 128 > len;
            if (diag || tail) {
#pragma unroll
                for (int e = 0; e < 128; ++e) {
                    const int kv = kv0 + e;
                    const bool valid = !(diag && kv > q_local) && kv < len;
                    sv[e] = valid ? sv[e] : -INFINITY;
                }
            }
            // row maximum of the raw scores (three-input maxima, four independent chains);
            // the scale is positive, so scaling the maximum gives the scaled maximum
            float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int e = 0; e < 128; e += 8) {
#pragma unroll
                for (int q = 0; q < 4; ++q) mq[q] = fmax3(mq[q], sv[e + 2 * q], sv[e + 2 * q + 1]);
            }
            const float mx = fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3])) * prm.scale_log2;
            // stale-max rule: keep the old reference unless the row maximum grew a lot
            float alpha = 1.f;
            bool rescale = false;
            if (j == 0) {
                m_ref = mx;
            } else if (mx > m_ref + kRescaleThreshold) {
                alpha = fast_exp2(m_ref - mx);
                m_ref = mx;
                rescale = true;
            }
            if (__any_sync(0xffffffffu, rescale)) {
                // O_t must hold the previous P.V product before it is rescaled (it does: S
                // of this step completed after it); no P.V of this step has started yet
                const bool got_o = mbar_wait_or_abort(&bar_o_done[t], (j - 1) & 1, 31, abort_flag);
                if (!__all_sync(0xffffffffu, got_o)) { failed = true; break; }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    float ov[32];
                    tmem_ld32(t_o + c * 32, ov);
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] *= alpha;
                    tmem_st32(t_o + c * 32, ov);
                }
            }
            // P = 2^(scale * S - m_ref), in four chunks of 32 columns, software-pipelined:
            // the exponentials of chunk c+1 are issued ahead of the row sums, the bf16
            // packing and the TMEM store of chunk c, so that one warp keeps the MUFU busy
            const float neg_m = -m_ref;
            // (scale and subtract, and the row sums, in packed pairs)
            const float2 sc2 = make_float2(prm.scale_log2, prm.scale_log2);
            const float2 nm2 = make_float2(neg_m, neg_m);
            auto exps = [&](int c, float (&p)[32]) {
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float2 x = f2_fma(make_float2(sv[c * 32 + e], sv[c * 32 + e + 1]), sc2, nm2);
                    p[e] = fast_exp2(x.x);
                    p[e + 1] = fast_exp2(x.y);
                }
            };
            float2 rsA = make_float2(0.f, 0.f), rsB = make_float2(0.f, 0.f);
            auto finish = [&](int c, const float (&p)[32]) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    if (e & 1)
                        rsB = f2_add(rsB, make_float2(p[2 * e], p[2 * e + 1]));
                    else
                        rsA = f2_add(rsA, make_float2(p[2 * e], p[2 * e + 1]));
                    pk[e] = pack_bf16(p[2 * e], p[2 * e + 1]);
                }
                tmem_st16(t_s + c * 16, pk);   // P (packed) over S columns already read
            };
            {
                float pa[32], pb[32];
                exps(0, pa);
                exps(1, pb);
                finish(0, pa);
                exps(2, pa);
                finish(1, pb);
                // the first half of P (columns [0, 64), K = 0..63 of P.V) is in TMEM
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bar_p_half[t]);
                exps(3, pb);
                finish(2, pa);
                finish(3, pb);
            }
            const float rs_all = (rsA.x + rsA.y) + (rsB.x + rsB.y);
            l_run = l_run * alpha + rs_all;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar_p_ready[t]);
        }
        // ---- epilogue: O / l -> bf16, LSE ----
        bool have = !failed && nk > 0 && !*abort_flag;
        if (have) have = mbar_wait_or_abort(&bar_o_done[t], (nk - 1) & 1, 32, abort_flag);
        have = __all_sync(0xffffffffu, have);
        if (have) {
            tc_fence_after();
            const bool row_ok = q_local < len;
            const float inv_l = 1.f / l_run;
            const int tok = seg0 + q_local;
            __nv_bfloat16* orow = prm.o + ((size_t)tok * prm.hq + h) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                float ov[32];
                tmem_ld32(t_o + c * 32, ov);
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
                prm.lse[(size_t)h * prm.T + tok] = (m_ref + __log2f(l_run)) * 0.69314718055994531f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace lf
