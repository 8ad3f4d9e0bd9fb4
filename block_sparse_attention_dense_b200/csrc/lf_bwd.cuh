// LazyFlash block-sparse attention backward on sm_100a (article sections "Le
// passage arrière fait deux fois le travail du passage avant" and "Un budget
// sur la masse de gradient, et un tirage qui garde le gradient non biaisé":
// only kept query blocks are loaded and computed, and their output gradient
// carries the weight 1/p).
//
// One CTA owns a 128-row KV tile j of one segment for up to four query heads of
// the same KV head (the whole query group when it has 1, 2 or 4 heads) and walks
// their kept query tiles t (t >= j when causal) from the compacted kept-block
// lists, head by head.  CTAs are ordered KV tile fastest, so the CTAs resident at
// any time share those heads: their Q, dO and fp32 dQ accumulators (about 128 MB
// for four heads at 32K tokens) stay largely in L2, where the dQ reductions run at
// L2 rather than HBM speed.  dK/dV sum the CTA's heads in TMEM; when the CTA holds
// the whole query group they are final and stored as bf16, otherwise each CTA's
// tile is added into fp32 accumulators by TMA reduce-adds (one per CTA, not per
// pair).  Each 128-row query tile is handled as two 64-column halves, so that the
// element-wise work on one half overlaps the tensor-core work on the other.
// Per half:
//   tcgen05 (SS): S^T  = K_j Q_h^T,  dP^T = V_j dO_h^T        (TMEM, fp32)
//   element-wise: P = exp2(S*scale*log2e - LSE*log2e), dS = P (dP - D), both
//                 times the block weight; P^T and dS^T rounded to bf16 back
//                 into TMEM (both over S^T) and dS^T into shared memory
//   tcgen05 (SS): dQ_h^T = K_j^T dS^T_h       (TMEM, over dP^T; lanes = d)
//   tcgen05 (TS): dV_j += P^T dO_h, dK_j += dS^T Q_h   (A from TMEM)
//   dQ drain:     lane d adds column q of dQ_h^T into the fp32 accumulator;
//                 a warp's 32 lanes hit 32 consecutive floats of one row.
// Roles (512 threads): warp 0 TMA producer and work list, warps 1 and 2 MMA
// issuers for query halves 0 and 1 (the whole warp runs it, one elected lane
// issues), warps 4-7 and 12-15 element-wise on columns [0, 32) and [32, 64) of
// each half (+ the dV and the dK epilogue respectively): thread = KV row = TMEM
// lane; warps 8-11 dQ drain (thread = head-dim index = TMEM lane).
//
// kHalves (64-row selection blocks): a query half is one block and is live when its
// weight is non-zero; a dropped block's half is neither loaded (a tile with one live
// half loads Q and dO in 64-row boxes) nor computed, and a half past the segment's end
// is skipped the same way.  Every role counts a half's barrier phases by its live
// pairs, and dV and dK start from zeros stored in TMEM, so the first gradient MMA of
// either half may come first.  With 128-row blocks both halves of a tile carry the
// same block's weight, and the kernel keeps one phase per pair (the skipping
// variant's bookkeeping cost about 4 % there, A/B on one GPU).
//
// Tensor memory (512 columns): dV [0,128) dK [128,256); half 0: S^T [256,320)
// (after the element-wise pass: P^T in its first 32 columns, dS^T in the next 32,
// both bf16 packed two per column), dP^T then dQ^T [320,384); half 1: [384,448),
// [448,512).  Reuse of a region by a later MMA relies on tcgen05.mma executing in
// issue order.
#pragma once

#include "lf_device.cuh"

namespace lf {

struct BwdParams {
    const int32_t* cu_seqlens;
    int T, hq, hkv, causal, block_q, nbmax, max_seqlen;
    int heads_per_cta;         // query heads of one KV head per CTA (<= kMaxHeadsPerCta)
    float scale;               // softmax_scale
    float scale_log2;          // softmax_scale * log2(e)
    const float* lse;          // [hq][T], natural log
    const float* Dvec;         // [hq][T]
    const float* block_weight; // [nseq][hq][nbmax]
    const int32_t* kept_idx;   // [nseq][hq][nbmax]
    const int32_t* kept_cnt;   // [nseq][hq]
    float* dq_acc;             // [hq][T][D] fp32 (head-major), zeroed by the caller
    // dK (unscaled) and dV go to [T][hkv][D] fp32 accumulators, zeroed by the caller,
    // through the tensor maps the kernel is given (32 x 1 x 128 boxes, 128-byte swizzle);
    // when a CTA covers the whole query group of its KV head (kv_out_direct) they go
    // instead, final, to the bf16 outputs [T][hkv][D], zeroed by the caller
    int kv_out_direct;
    // CTA order within a segment: 0 = KV tile fastest, one head group after another;
    // 1 = head group fastest (every group's heavy low tiles start first)
    int tile_major;
    __nv_bfloat16* dk_out;
    __nv_bfloat16* dv_out;
};

constexpr uint32_t kAccBox = 128 * 32 * 4;   // one staged 32-column fp32 box of a KV tile
constexpr int kMaxHeadsPerCta = 32;           // query heads one backward CTA can walk

template <int D>
struct BwdSmem {
    static constexpr int kPanels = D / 64;
    static constexpr uint32_t kTile = kPanels * kPanelBytes;   // 128 x D bf16
    static constexpr uint32_t kHalfDS = 128 * 128;             // [128 kv][64 q] bf16
    static constexpr uint32_t kK = 0;
    static constexpr uint32_t kV = kK + kTile;
    static constexpr uint32_t kQdo = kV + kTile;               // stage s: Q at +2s*kTile, dO at +(2s+1)*kTile
    static constexpr uint32_t kDS = kQdo + 4 * kTile;          // two halves
    static constexpr uint32_t kVec = kDS + 2 * kHalfDS;        // lse*log2e [128], D [128]
    static constexpr uint32_t kBars = kVec + 2 * 128 * 4;
    static constexpr uint32_t kHeads = kBars + 256;            // int2 per query head of the CTA
    static constexpr uint32_t kBytes = kHeads + kMaxHeadsPerCta * 8;
    static constexpr uint32_t kAlloc = kBytes + 1024;
};

constexpr int kBwdThreads = 512;

// One (query head, query tile) pair of a KV tile's walk, published by the
// producer warp so that no other role reads the kept lists from global memory.
// h < 0 marks the end of the walk.
struct PairEntry {
    int h, tile;
    float w0, w1;   // block weights of the tile's two 64-row halves
};

// First index i in list[0, cnt) with list[i] >= key (the list ascends), found by
// the whole warp: each round probes 32 evenly spaced entries at once and keeps the
// bracket between the last one below the key and the first one at or above it, so
// a list of up to 1024 entries takes two rounds of loads instead of ten dependent
// ones.  Every lane must call it and gets the same answer.
__device__ __forceinline__ int lower_bound_warp(const int32_t* list, int cnt, int key) {
    const int lane = threadIdx.x & 31;
    int lo = 0, hi = cnt;
    while (lo < hi) {
        const int step = (hi - lo + 31) >> 5;
        const int i = lo + lane * step;
        const unsigned below = __ballot_sync(0xffffffffu, i < hi && list[i] < key);
        const int nb = __popc(below);     // the probes below the key form a prefix
        const int new_hi = min(hi, lo + nb * step);
        lo = nb == 0 ? lo : lo + (nb - 1) * step + 1;
        hi = nb == 0 ? lo : new_hi;
    }
    return lo;
}

// Before the walk, the warps of the CTA find, head by head (warp w takes heads w,
// w + 16, ...), each head's first kept block at or after the CTA's first query tile
// with the warp-parallel search, and store (position, count) in shared memory; the
// return value says whether that head has any tile to visit (the same on every lane).
__device__ __forceinline__ bool find_head_starts(const BwdParams& p, int G, int g, int s, int jt,
                                                 int len, int2* heads) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int first_block = p.causal ? (jt * 128) / p.block_q : 0;
    const int nb = (len + p.block_q - 1) / p.block_q;
    bool any = false;
    for (int hh = warp; hh < G; hh += kBwdThreads / 32) {
        const int h = g * G + hh;
        const int32_t* l = p.kept_idx + ((size_t)s * p.hq + h) * p.nbmax;
        const int c = min(max(p.kept_cnt[(size_t)s * p.hq + h], 0), p.nbmax);
        const int start = first_block == 0 ? 0 : lower_bound_warp(l, c, first_block);
        if (lane == 0) heads[hh] = make_int2(start, c);
        if (start < c) {
            const int b = l[start];
            any = any || (b >= 0 && b < nb);
        }
    }
    return any;
}

// Walks the kept query tiles of heads g*G .. g*G+G-1 of one segment in ascending
// order of (head, tile), from the starts find_head_starts left in shared memory.
// Used by one thread (the producer).
struct KeptTileWalk {
    const int32_t* kept_idx;
    const int2* heads;
    int nbmax, hq, G, g, s, block_q, nb;
    int hh, pos, cnt;
    const int32_t* list;
    int tile, h;

    __device__ void init(const BwdParams& p, const int2* heads_, int G_, int g_, int s_, int len) {
        kept_idx = p.kept_idx;
        heads = heads_;
        nbmax = p.nbmax;
        hq = p.hq;
        G = G_;
        g = g_;
        s = s_;
        block_q = p.block_q;
        nb = (len + p.block_q - 1) / p.block_q;
    }
    __device__ void open_head() {
        h = g * G + hh;
        list = kept_idx + ((size_t)s * hq + h) * nbmax;
        const int2 e = heads[hh];
        pos = e.x;
        cnt = e.y;
    }
    // Moves to the next tile; returns false when the walk is over.
    __device__ bool next(bool first) {
        if (first) {
            hh = 0;
            open_head();
        } else {
            // skip the other blocks of the tile just processed
            while (pos < cnt && (list[pos] * block_q) / 128 == tile) ++pos;
        }
        for (;;) {
            while (pos >= cnt) {
                if (++hh >= G) return false;
                open_head();
            }
            const int b = list[pos];
            if (b >= 0 && b < nb) {
                tile = (b * block_q) / 128;
                return true;
            }
            pos = cnt;   // an entry outside the segment ends this head's walk
        }
    }
};

// Weight of the query rows [q0, q0 + 64) of a tile (one selection block, or
// half of one): 0 past the segment's end.
__device__ __forceinline__ float half_weight(const BwdParams& p, int s, int h, int q0, int len) {
    if (q0 >= len) return 0.f;
    return p.block_weight[((size_t)s * p.hq + h) * p.nbmax + q0 / p.block_q];
}

template <int D, bool kHalves>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dvacc, const __grid_constant__ CUtensorMap tm_dkacc,
                    const __grid_constant__ CUtensorMap tm_q64, const __grid_constant__ CUtensorMap tm_do64,
                    BwdParams prm) {
    using L = BwdSmem<D>;
    static_assert(2 * (D / 32) * kAccBox <= 4 * L::kTile, "dK/dV staging must fit the Q/dO buffers");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* lse2_s = reinterpret_cast<float*>(smem + L::kVec);   // -LSE * log2(e) per column
    float* dvec_s = lse2_s + 128;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
    uint64_t* bar_kv = bars + 0;
    uint64_t* bar_qdo_full = bars + 1;    // [2] stages
    uint64_t* bar_qdo_empty = bars + 3;   // [2]
    uint64_t* bar_s_full = bars + 5;      // [2] halves
    uint64_t* bar_p_ready = bars + 7;     // [2]
    uint64_t* bar_dq_full = bars + 9;     // [2]
    uint64_t* bar_dq_free = bars + 11;    // [2]
    uint64_t* bar_done = bars + 13;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 15);
    uint64_t* bar_entry = bars + 16;      // [4] work-list ring
    PairEntry* ring = reinterpret_cast<PairEntry*>(bars + 20);   // [4] x 16 B
    uint64_t* bar_acc0 = bars + 28;       // one phase: half 0's first dV/dK MMAs completed (!kHalves)

    // KV tile fastest: CTAs resident together share one head group, so its Q, dO and
    // dQ accumulator stay in L2, and each group's lowest tiles (most work) start first.
    // When a segment's CTAs make only a few waves, the last group's heaviest CTAs would
    // start late and run alone at the end; there the group runs fastest instead, so
    // that the heavy tiles of every group start first.
    int jt, hgrp;                           // hgrp: query heads hgrp*G .. hgrp*G+G-1, G = heads_per_cta
    if (prm.tile_major) {
        const int lin = static_cast<int>(blockIdx.x + blockIdx.y * gridDim.x);
        jt = lin / static_cast<int>(gridDim.y);
        hgrp = lin % static_cast<int>(gridDim.y);
    } else {
        jt = blockIdx.x;
        hgrp = blockIdx.y;
    }
    const int s = blockIdx.z;
    int seg0, len;
    if (!load_segment(prm.cu_seqlens, s, prm.T, prm.max_seqlen, seg0, len, 30)) return;
    if (jt * 128 >= len) return;
    const int g = hgrp * prm.heads_per_cta / (prm.hq / prm.hkv);   // their KV head

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t s_base = smem_addr(smem);

    if (tid == 0) {
        mbar_init(bar_kv, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_qdo_full[i], 1);
            mbar_init(&bar_qdo_empty[i], 2);   // one commit per MMA issuer
            mbar_init(&bar_s_full[i], 1);
            mbar_init(&bar_p_ready[i], 256);
            mbar_init(&bar_dq_full[i], 1);
            mbar_init(&bar_dq_free[i], 128);
        }
        mbar_init(bar_done, 2);                 // one commit per MMA issuer
        for (int i = 0; i < 4; ++i) mbar_init(&bar_entry[i], 1);
        mbar_init(bar_acc0, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_do);
        prefetch_tensormap(&tm_dvacc);
        prefetch_tensormap(&tm_dkacc);
        prefetch_tensormap(&tm_q64);
        prefetch_tensormap(&tm_do64);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    // every head's first kept tile for this KV tile; does the tile have any work?
    int2* head_starts = reinterpret_cast<int2*>(smem + L::kHeads);
    const bool has = find_head_starts(prm, prm.heads_per_cta, hgrp, s, jt, len, head_starts);
    tc_fence_before();
    const bool any = __syncthreads_or(has) != 0;   // the same answer in every role
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_dv = tmem;
    const uint32_t t_dk = tmem + 128;
    const int kv_row0 = seg0 + jt * 128;

    KeptTileWalk walk;
    walk.init(prm, head_starts, prm.heads_per_cta, hgrp, s, len);

    constexpr uint32_t kIdescS = idesc_bf16(128, 64, 0, 0);    // S^T, dP^T halves
    constexpr uint32_t kIdescKV = idesc_bf16(128, D, 0, 1);    // dV, dK (A from TMEM, B MN-major)
    constexpr uint32_t kIdescQ = idesc_bf16(128, 64, 1, 1);    // dQ^T half (A K^T, B dS^T: MN-major)

    if (warp == 0) {
        // ===================== TMA producer + work list =====================
        if (lane == 0) {
            uint32_t fill_parity[2] = {0, 0};
            bool filled[2] = {false, false};
            if (any) {
                mbar_arrive_expect_tx(bar_kv, 2 * L::kTile);
                for (int c = 0; c < L::kPanels; ++c) {
                    tma_load_3d(smem + L::kK + c * kPanelBytes, &tm_k, bar_kv, c * 64, g, kv_row0);
                    tma_load_3d(smem + L::kV + c * kPanelBytes, &tm_v, bar_kv, c * 64, g, kv_row0);
                }
            }
            int n = 0;
            bool more = any && walk.next(true), ok = true;
            while (more) {
                const int st = n & 1;
                // the stage (and, by the pipeline's order, ring slot n % 4) is free
                if (n >= 2 && !mbar_wait_or_abort(&bar_qdo_empty[st], ((n >> 1) - 1) & 1, 31, abort_flag)) {
                    ok = false;
                    break;
                }
                const int q0 = walk.tile * 128;
                PairEntry e;
                e.h = walk.h;
                e.tile = walk.tile;
                e.w0 = half_weight(prm, s, walk.h, q0, len);
                e.w1 = half_weight(prm, s, walk.h, q0 + 64, len);
                ring[n & 3] = e;
                mbar_arrive(&bar_entry[n & 3]);
                // Q and dO rows of the tile's live halves only: both halves in 128-row boxes,
                // a single live half in 64-row boxes; a half whose block was dropped, or that
                // lies past the segment's end, is not loaded
                const bool live0 = !kHalves || e.w0 != 0.f, live1 = !kHalves || e.w1 != 0.f;
                const uint32_t nlive = (live0 ? 1u : 0u) + (live1 ? 1u : 0u);
                mbar_arrive_expect_tx(&bar_qdo_full[st], nlive * L::kTile);
                const int hh = live0 ? 0 : 1;                     // the single live half
                const CUtensorMap* mq = nlive == 2 ? &tm_q : &tm_q64;
                const CUtensorMap* mdo = nlive == 2 ? &tm_do : &tm_do64;
                const int row = seg0 + q0 + (nlive == 2 ? 0 : 64 * hh);
                const uint32_t off = nlive == 2 ? 0u : hh * 8192u;
                for (int c = 0; c < L::kPanels; ++c) {
                    tma_load_3d(smem + L::kQdo + (2 * st) * L::kTile + c * kPanelBytes + off, mq,
                                &bar_qdo_full[st], c * 64, walk.h, row);
                    tma_load_3d(smem + L::kQdo + (2 * st + 1) * L::kTile + c * kPanelBytes + off, mdo,
                                &bar_qdo_full[st], c * 64, walk.h, row);
                }
                fill_parity[st] = (n >> 1) & 1;
                filled[st] = true;
                ++n;
                more = walk.next(false);
            }
            // end-of-walk entry (slot n % 4 was last used by pair n - 4)
            if (ok && n >= 2 &&
                !mbar_wait_or_abort(&bar_qdo_empty[n & 1], ((n >> 1) - 1) & 1, 31, abort_flag))
                ok = false;
            if (ok) {
                PairEntry e;
                e.h = -1;
                e.tile = 0;
                e.w0 = e.w1 = 0.f;
                ring[n & 3] = e;
                mbar_arrive(&bar_entry[n & 3]);
            }
            if (*abort_flag) {
                // let this CTA's own copies land before the CTA exits (bounded)
                if (any) mbar_wait(bar_kv, 0, 32);
                for (int st = 0; st < 2; ++st)
                    if (filled[st]) mbar_wait(&bar_qdo_full[st], fill_parity[st], 32);
            }
        }
        __syncwarp();
    } else if (warp == 1 || warp == 2) {
        // ============ MMA issuers: warp 1 for query half 0, warp 2 for half 1 ============
        // Each issuer runs its half's chain (S^T/dP^T -> element-wise -> dV, dK, dQ^T ->
        // drain -> next S^T/dP^T) on its own, so one half's waits overlap the other
        // half's MMAs.  The whole warp runs the code and one elected lane issues; every
        // wait result is warp-uniform, and each commit tracks its issuing lane's MMAs.
        const int hf = warp - 1;
        if (any) {
            auto wait = [&](uint64_t* bar, uint32_t parity, int site) {
                return __all_sync(0xffffffffu, mbar_wait_or_abort(bar, parity, site, abort_flag));
            };
            const uint32_t ka = s_base + L::kK, va = s_base + L::kV;
            auto stage_q = [&](int n) { return s_base + L::kQdo + (2 * (n & 1)) * L::kTile; };
            const uint32_t t_s = tmem + 256 + hf * 128, t_dp = t_s + 64;
            // S^T of one half of pair n (into the S^T columns)
            auto issue_s = [&](int n) {
                const uint32_t qa = stage_q(n);
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    mma_bf16_ss_warp(t_s, desc_kmajor(ka, k), desc_kmajor(qa + hf * 8192, k), kIdescS, k > 0);
            };
            // dP^T of one half of pair n (into the dP^T columns), then the commit that
            // hands S^T and dP^T to the element-wise warps
            auto issue_dp = [&](int n) {
                const uint32_t da = stage_q(n) + L::kTile;
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    mma_bf16_ss_warp(t_dp, desc_kmajor(va, k), desc_kmajor(da + hf * 8192, k), kIdescS, k > 0);
                mma_commit_warp(&bar_s_full[hf]);
            };
            // dQ^T (SS, into the dP^T columns, which the element-wise pass has read) first,
            // so that the drain can start; then dV and dK (TS: P^T and dS^T from the S^T
            // columns)
            auto issue_grads = [&](int n) {
                const uint32_t qa = stage_q(n), da = qa + L::kTile;
                const uint32_t dsa = s_base + L::kDS + hf * L::kHalfDS;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    // A = K^T (M = d): MN-major over the K tile; with d = 64 the
                    // second 64-row atom repeats the first (those lanes are unused)
                    const uint64_t adesc =
                        (D == 128) ? desc_mnmajor(ka, k) : sw128_desc(ka + k * 2048, 0, 1024);
                    mma_bf16_ss_warp(t_dp, adesc, desc_mnmajor(dsa, k), kIdescQ, k > 0);
                }
                mma_commit_warp(&bar_dq_full[hf]);
                // kHalves: dV and dK accumulate onto TMEM the element-wise warps zeroed at
                // the start; otherwise half 0's first ones start them
                const uint32_t first = (kHalves || n > 0 || hf > 0) ? 1u : 0u;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16_ts_warp(t_dv, t_s + k * 8, desc_mnmajor(da, hf * 4 + k), kIdescKV,
                                     (first || k > 0) ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16_ts_warp(t_dk, t_s + 32 + k * 8, desc_mnmajor(qa, hf * 4 + k), kIdescKV,
                                     (first || k > 0) ? 1u : 0u);
                mma_commit_warp(&bar_qdo_empty[n & 1]);   // this half is done with the Q/dO stage
            };
            // Order per half: S^T of the next pair goes out right after this half's gradients
            // (the pipe runs it after dV and dK have read P^T and dS^T from those columns);
            // its dP^T as soon as the half's last dQ^T has been drained from the dP^T
            // columns.  A pair whose half is not live (its 64-row block dropped, or past the
            // segment's end) is skipped by every role of that half: the half's barriers
            // count live pairs (kg), and only the Q/dO stage is released for it.
            if constexpr (kHalves) {
                auto live = [&](const PairEntry& x) { return (hf ? x.w1 : x.w0) != 0.f; };
                int kg = 0;                  // this half's live pairs whose gradients are issued
                bool pending_free = false;   // the last dQ^T still occupies the dP^T columns
                bool have = wait(bar_kv, 0, 33) && wait(&bar_entry[0], 0, 34);
                PairEntry cur = ring[0];
                have = have && cur.h >= 0;
                if (have && live(cur)) {
                    have = wait(&bar_qdo_full[0], 0, 34);
                    if (have) {
                        tc_fence_after();
                        issue_s(0);
                        issue_dp(0);
                    }
                }
                for (int n = 0; have; ++n) {
                    if (!wait(&bar_entry[(n + 1) & 3], ((n + 1) >> 2) & 1, 34)) break;
                    const PairEntry nxt = ring[(n + 1) & 3];
                    if (live(cur)) {
                        if (!wait(&bar_p_ready[hf], kg & 1, 36)) break;
                        tc_fence_after();
                        issue_grads(n);
                        ++kg;
                        pending_free = true;
                    } else {
                        mma_commit_warp(&bar_qdo_empty[n & 1]);   // nothing of this half reads the stage
                    }
                    if (nxt.h < 0) break;
                    if (live(nxt)) {
                        if (!wait(&bar_qdo_full[(n + 1) & 1], ((n + 1) >> 1) & 1, 34)) break;
                        tc_fence_after();
                        issue_s(n + 1);
                        if (pending_free) {
                            if (!wait(&bar_dq_free[hf], (kg - 1) & 1, 35)) break;
                            pending_free = false;
                            tc_fence_after();
                        }
                        issue_dp(n + 1);
                    }
                    cur = nxt;
                }
            } else {
                // one phase per pair: dV and dK collect both halves in pipe order, so half
                // 1's first gradients wait until half 0's first ones (which start the
                // accumulators) have completed
                bool have = wait(bar_kv, 0, 33) && wait(&bar_entry[0], 0, 34);
                have = have && ring[0].h >= 0 && wait(&bar_qdo_full[0], 0, 34);
                if (have) {
                    tc_fence_after();
                    issue_s(0);
                    issue_dp(0);
                }
                for (int n = 0; have; ++n) {
                    if (!wait(&bar_entry[(n + 1) & 3], ((n + 1) >> 2) & 1, 34)) break;
                    const bool next = ring[(n + 1) & 3].h >= 0;
                    if (!wait(&bar_p_ready[hf], n & 1, 36)) break;
                    if (hf == 1 && n == 0 && !wait(bar_acc0, 0, 44)) break;
                    tc_fence_after();
                    issue_grads(n);
                    if (hf == 0 && n == 0) mma_commit_warp(bar_acc0);
                    if (!next) break;
                    if (!wait(&bar_qdo_full[(n + 1) & 1], ((n + 1) >> 1) & 1, 34)) break;
                    tc_fence_after();
                    issue_s(n + 1);
                    if (!wait(&bar_dq_free[hf], n & 1, 35)) break;
                    tc_fence_after();
                    issue_dp(n + 1);
                }
            }
            mma_commit_warp(bar_done);
            // every MMA this warp issued must finish before TMEM is released
            __all_sync(0xffffffffu, mbar_wait(bar_done, 0, 37));
        }
    } else if ((warp >= 4 && warp < 8) || warp >= 12) {
        // ===== element-wise: both warpgroups on each half, 32 columns each (thread = KV row) =====
        const int wg = warp >= 12 ? 1 : 0;                // columns [32 wg, 32 wg + 32) of a half
        const int hf_epi = wg;                            // epilogue: 0 -> dV, 1 -> dK
        const int r = (warp & 3) * 32 + lane;             // TMEM lane / KV row
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int kv_local = jt * 128 + r;
        const bool kv_valid = kv_local < len;
        // P = 0 where kv_cmp > the query's index: the key follows the query (causal), or
        // the KV row lies past the segment's end (its key belongs to the next segment, so
        // its exponent is not bounded by this query's LSE and must not reach the products)
        const int kv_cmp = !kv_valid ? 0x7fffffff : (prm.causal ? kv_local : (int)0x80000000);
        int n = 0;
        // parity of each half's live pairs processed (bit hf: the half's barrier phase);
        // bits of one register rather than an array indexed by the half loop, which would
        // live in local memory
        uint32_t ke = 0;
        bool more = any, failed = false;
        if (kHalves && any) {
            // dV (warpgroup 0) and dK (warpgroup 1) start from zero in TMEM, so that every
            // gradient MMA accumulates, whichever half and pair comes first; the stores are
            // complete before this warpgroup's first p_ready arrival
            const uint32_t t_acc = (wg ? t_dk : t_dv) + lane_off;
            float z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) z[i] = 0.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) tmem_st32(t_acc + c * 32, z);
            tmem_wait_st();
        }
        for (;;) {
            // uniform decision of both warpgroups; also: all are done with the old vectors
            if (named_bar_or(1, 256, !more || failed)) break;
            const bool got_e = mbar_wait_or_abort(&bar_entry[n & 3], (n >> 2) & 1, 41, abort_flag);
            const PairEntry e = ring[n & 3];
            if (!got_e || e.h < 0) {
                more = false;
                failed = !got_e;
                continue;
            }
            const int qt = e.tile, q0 = qt * 128;
            if (r < 64) {
                // this warpgroup's 64 columns: [32 wg, 32 wg + 32) of each half
                const int col = (r >> 5) * 64 + wg * 32 + (r & 31);
                const int q_local = q0 + col;
                float l2 = INFINITY, dd = 0.f;    // exp2(S - inf) = 0: columns past the segment vanish
                if (q_local < len) {
                    const size_t idx = (size_t)e.h * prm.T + seg0 + q_local;
                    l2 = prm.lse[idx] * 1.4426950408889634f;
                    dd = prm.Dvec[idx];
                }
                lse2_s[col] = -l2;   // stored negated: the exponent is one packed FMA
                dvec_s[col] = dd;
            }
            named_bar_sync(2, 256);
            for (int hf = 0; hf < 2; ++hf) {
                const float w = hf ? e.w1 : e.w0;
                if (kHalves && w == 0.f) continue;   // not live: nothing was loaded or computed for it
                const uint32_t t_s = tmem + 256 + hf * 128 + lane_off, t_dp = t_s + 64;
                const uint32_t dsa = s_base + L::kDS + hf * L::kHalfDS;
                const uint32_t par = kHalves ? (ke >> hf) & 1u : static_cast<uint32_t>(n & 1);
                const bool got = mbar_wait_or_abort(&bar_s_full[hf], par, 38, abort_flag);
                const bool ok = __all_sync(0xffffffffu, got);
                // this warpgroup's two 16-column chunks of S^T and dP^T
                uint32_t sa[16], da[16], sb[16], db[16];
                if (ok) {
                    tc_fence_after();
                    tmem_ld16_nowait(t_s + (2 * wg) * 16, sa);
                    tmem_ld16_nowait(t_dp + (2 * wg) * 16, da);
                    tmem_ld16_nowait(t_s + (2 * wg + 1) * 16, sb);
                    tmem_ld16_nowait(t_dp + (2 * wg + 1) * 16, db);
                    tmem_wait_ld_regs(sa, da);
                    tmem_wait_ld_regs(sb, db);
                }
                // every fp32 column of the half is in registers before P^T/dS^T are
                // written over them (the packed columns of one warpgroup overlap the
                // fp32 columns of the other)
                named_bar_sync(3, 256);
                if (!ok) { failed = true; continue; }
                auto chunk = [&](int c, const uint32_t (&sr)[16], const uint32_t (&dr)[16]) {
                    uint32_t pk[8], dk_[8];
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const int col0 = hf * 64 + c * 16 + 4 * e4;
                        const float4 l4 = *reinterpret_cast<const float4*>(lse2_s + col0);
                        const float4 d4 = *reinterpret_cast<const float4*>(dvec_s + col0);
                        const float2 sc2 = make_float2(prm.scale_log2, prm.scale_log2);
                        const float2 w2 = make_float2(w, w);
                        float pw[4], dsw[4];
                        // two columns per packed instruction
#pragma unroll
                        for (int u = 0; u < 4; u += 2) {
                            const float2 nl = u ? make_float2(l4.z, l4.w) : make_float2(l4.x, l4.y);
                            const float2 dv2 = u ? make_float2(d4.z, d4.w) : make_float2(d4.x, d4.y);
                            const float2 s2 = make_float2(__uint_as_float(sr[4 * e4 + u]),
                                                          __uint_as_float(sr[4 * e4 + u + 1]));
                            const float2 dp2 = make_float2(__uint_as_float(dr[4 * e4 + u]),
                                                           __uint_as_float(dr[4 * e4 + u + 1]));
                            const float2 x = f2_fma(s2, sc2, nl);
                            float p0 = fast_exp2(x.x), p1 = fast_exp2(x.y);
                            if (kv_cmp > q0 + col0 + u) p0 = 0.f;
                            if (kv_cmp > q0 + col0 + u + 1) p1 = 0.f;
                            const float2 pw2 = f2_mul(make_float2(p0, p1), w2);
                            const float2 ds2 = f2_mul(pw2, f2_sub(dp2, dv2));
                            pw[u] = pw2.x;
                            pw[u + 1] = pw2.y;
                            dsw[u] = ds2.x;
                            dsw[u + 1] = ds2.y;
                        }
                        pk[2 * e4] = pack_bf16(pw[0], pw[1]);
                        pk[2 * e4 + 1] = pack_bf16(pw[2], pw[3]);
                        dk_[2 * e4] = pack_bf16(dsw[0], dsw[1]);
                        dk_[2 * e4 + 1] = pack_bf16(dsw[2], dsw[3]);
                    }
                    tmem_st8(t_s + c * 8, pk);          // P^T, packed columns [8c, 8c+8)
                    tmem_st8(t_s + 32 + c * 8, dk_);    // dS^T, packed columns [32 + 8c, ...)
                    st_shared_v4(dsa + sw128_chunk_offset(r, 2 * c), dk_[0], dk_[1], dk_[2], dk_[3]);
                    st_shared_v4(dsa + sw128_chunk_offset(r, 2 * c + 1), dk_[4], dk_[5], dk_[6], dk_[7]);
                };
                chunk(2 * wg, sa, da);
                chunk(2 * wg + 1, sb, db);
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bar_p_ready[hf]);
                ke ^= 1u << hf;
            }
            if (!failed) ++n;
        }
        // ---- epilogue: warpgroup 0 adds dV, warpgroup 1 adds dK (unscaled) into the
        // fp32 accumulators of the KV head (the GQA sum over query heads).  Each thread
        // stages its KV row in the Q/dO buffers, free once every MMA has completed, as
        // 32-column boxes with the 128-byte swizzle; one thread then adds the boxes with
        // TMA reduce-adds (rows past the segment's end hold exact zeros: P and dS are
        // 0 there; rows past the tensor's end are clipped by the copy) ----
        bool have = n > 0 && !failed && !*abort_flag;
        if (have) have = mbar_wait_or_abort(bar_done, 0, 39, abort_flag) && !*abort_flag;
        // one decision per warpgroup: all 128 threads meet at the staging barrier
        have = !named_bar_or(6 + wg, 128, !have);
        if (have && prm.kv_out_direct) {
            // the CTA holds its KV head's whole query group: the tile is final, so it
            // goes straight to the bf16 output (dK takes the softmax scale); rows past
            // the segment's end belong to the next segment and are not written
            tc_fence_after();
            const uint32_t t_acc = (hf_epi ? t_dk : t_dv) + lane_off;
            const float sc = hf_epi ? prm.scale : 1.f;
            __nv_bfloat16* dst = (hf_epi ? prm.dk_out : prm.dv_out) + ((size_t)(kv_row0 + r) * prm.hkv + g) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                float v[32];
                tmem_ld32(t_acc + c * 32, v);
                uint32_t pk[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) pk[k] = pack_bf16(v[2 * k] * sc, v[2 * k + 1] * sc);
                if (kv_valid) {
                    uint4* o = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        o[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                }
            }
        } else if (have) {
            tc_fence_after();
            const uint32_t t_acc = (hf_epi ? t_dk : t_dv) + lane_off;
            uint8_t* stage = smem + L::kQdo + hf_epi * (D / 32) * kAccBox;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                float v[32];
                tmem_ld32(t_acc + c * 32, v);
                const uint32_t row = smem_addr(stage + c * kAccBox) + r * 128;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    st_shared_v4(row + ((k ^ (r & 7)) << 4), __float_as_uint(v[4 * k]),
                                 __float_as_uint(v[4 * k + 1]), __float_as_uint(v[4 * k + 2]),
                                 __float_as_uint(v[4 * k + 3]));
            }
            fence_proxy_async_smem();
            named_bar_sync(6 + wg, 128);
            if (r == 0) {
                const CUtensorMap* map = hf_epi ? &tm_dkacc : &tm_dvacc;
                for (int c = 0; c < D / 32; ++c)
                    tma_reduce_add_3d(map, stage + c * kAccBox, 32 * c, g, kv_row0);
                bulk_commit_group();
                bulk_wait0();   // added (and the staging read) before the CTA exits
            }
        }
    } else if (warp >= 8 && warp < 12) {
        // ===================== dQ drain (thread = head-dim index) =====================
        const int dd = tid - 256;                         // TMEM lane = d index
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const bool lane_used = (warp & 3) * 32 < D;       // d = 64: warps 10, 11 idle
        int n = 0;
        uint32_t kd = 0;      // parity of each half's live pairs drained (bit hf)
        bool more = any;
        while (more) {
            const bool got_e = mbar_wait_or_abort(&bar_entry[n & 3], (n >> 2) & 1, 42, abort_flag);
            if (!__all_sync(0xffffffffu, got_e)) break;
            const PairEntry e = ring[n & 3];
            if (e.h < 0) break;
            const int q0 = e.tile * 128;
            bool ok = true;
            for (int hf = 0; hf < 2; ++hf) {
                if (kHalves && (hf ? e.w1 : e.w0) == 0.f) continue;   // not live: no dQ^T for this half
                const uint32_t par = kHalves ? (kd >> hf) & 1u : static_cast<uint32_t>(n & 1);
                const bool got = mbar_wait_or_abort(&bar_dq_full[hf], par, 40, abort_flag);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                kd ^= 1u << hf;
                tc_fence_after();
                const int qh = q0 + hf * 64;
                const bool live = lane_used && qh < len && (kHalves || (hf ? e.w1 : e.w0) != 0.f);
                // copy the half's dQ^T to registers and hand its TMEM columns back to
                // the MMA issuer at once; the reductions follow off its critical path
                float v[64];
                if (live) {
                    const uint32_t t_q = tmem + 256 + hf * 128 + 64 + lane_off;   // dP^T columns
                    uint32_t a[16], b[16];
#pragma unroll
                    for (int c = 0; c < 4; c += 2) {
                        tmem_ld16_nowait(t_q + c * 16, a);
                        tmem_ld16_nowait(t_q + (c + 1) * 16, b);
                        tmem_wait_ld_regs(a, b);
#pragma unroll
                        for (int e2 = 0; e2 < 16; ++e2) {
                            v[c * 16 + e2] = __uint_as_float(a[e2]);
                            v[(c + 1) * 16 + e2] = __uint_as_float(b[e2]);
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&bar_dq_free[hf]);
                if (live) {
                    // head-major accumulator: the half's 64 query rows are contiguous
                    float* dst = prm.dq_acc + ((size_t)e.h * prm.T + seg0 + qh) * D + dd;
                    const int nvalid = min(64, len - qh);
#pragma unroll
                    for (int q = 0; q < 64; ++q)
                        if (q < nvalid) atomicAdd(dst + q * D, v[q]);
                }
            }
            if (!ok) break;
            ++n;
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
