// LazyFlash block-sparse attention backward on sm_100a (article sections "Le
// passage arrière fait deux fois le travail du passage avant" and "Un budget
// sur la masse de gradient, et un tirage qui garde le gradient non biaisé":
// only kept query blocks are loaded and computed, and their output gradient
// carries the weight 1/p).
//
// One CTA owns a 128-row KV tile j of one KV head g of one segment and walks,
// for every query head of g's group, the kept query tiles t (t >= j when
// causal) from the compacted kept-block lists.  Per (t, j) pair:
//   tcgen05:  S^T  = K_j Q_t^T           (TMEM, 128 KV lanes x 128 q cols)
//             dP^T = V_j dO_t^T          (TMEM)
//   4 warps:  thread r owns KV row r:  P = exp2(S * scale*log2e - LSE*log2e),
//             dS = P (dP - D), both times the column's block weight, rounded
//             to bf16 into shared memory (K-major over q)
//   tcgen05:  dV_j += P^T dO_t, dK_j += dS^T Q_t   (TMEM, accumulated over the
//             whole walk: no atomics for dK/dV), dQ_t(partial) = dS K_j (TMEM)
//   4 warps:  thread r now owns query row r of the partial dQ and adds it into
//             the fp32 dQ accumulator (vector atomics).
// The epilogue writes dK (times softmax_scale) and dV as bf16; a KV tile that
// no kept block reaches gets zeros.
#pragma once

#include "lf_device.cuh"

namespace lf {

struct BwdParams {
    const int32_t* cu_seqlens;
    int T, hq, hkv, causal, block_q, nbmax, max_seqlen;
    float scale;               // softmax_scale
    float scale_log2;          // softmax_scale * log2(e)
    const float* lse;          // [hq][T], natural log
    const float* Dvec;         // [hq][T]
    const float* block_weight; // [nseq][hq][nbmax]
    const int32_t* kept_idx;   // [nseq][hq][nbmax]
    const int32_t* kept_cnt;   // [nseq][hq]
    float* dq_acc;             // [T][hq][D] fp32, zeroed by the caller
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
};

template <int D>
struct BwdSmem {
    static constexpr int kPanels = D / 64;
    static constexpr uint32_t kTile = kPanels * kPanelBytes;   // 128 x D bf16
    static constexpr uint32_t kK = 0;
    static constexpr uint32_t kV = kK + kTile;
    static constexpr uint32_t kQ = kV + kTile;
    static constexpr uint32_t kDO = kQ + kTile;
    static constexpr uint32_t kPt = kDO + kTile;               // 128 x 128 bf16
    static constexpr uint32_t kDSt = kPt + 2 * kPanelBytes;    // 128 x 128 bf16
    static constexpr uint32_t kVec = kDSt + 2 * kPanelBytes;   // lse2, D, w: 3 x 128 fp32
    static constexpr uint32_t kBars = kVec + 3 * 128 * 4;
    static constexpr uint32_t kBytes = kBars + 64;
    static constexpr uint32_t kAlloc = kBytes + 1024;
};

constexpr int kBwdThreads = 128;

// Walks the kept query tiles of one (segment, KV head) group in ascending order
// of (head in group, tile).  Every thread runs the same walk.
struct KeptTileWalk {
    const int32_t* kept_idx;
    const int32_t* kept_cnt;
    int nbmax, hq, G, g, s, block_q, first_block, nb;
    int hh, pos, cnt;
    const int32_t* list;
    int tile, h;

    __device__ void open_head() {
        h = g * G + hh;
        const size_t base = ((size_t)s * hq + h) * nbmax;
        list = kept_idx + base;
        cnt = min(max(kept_cnt[(size_t)s * hq + h], 0), nbmax);
        // first kept block >= first_block (lists are ascending)
        int lo = 0, hi = cnt;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (list[mid] < first_block) lo = mid + 1; else hi = mid;
        }
        pos = lo;
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

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    BwdParams prm) {
    using L = BwdSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* lse2_s = reinterpret_cast<float*>(smem + L::kVec);
    float* dvec_s = lse2_s + 128;
    float* w_s = dvec_s + 128;
    uint64_t* bar_kv = reinterpret_cast<uint64_t*>(smem + L::kBars);
    uint64_t* bar_qdo = bar_kv + 1;
    uint64_t* bar_mma = bar_kv + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_kv + 3);
    int* abort_flag = reinterpret_cast<int*>(bar_kv + 4);

    const int g = blockIdx.x;
    const int jt = blockIdx.y;              // KV tile: lowest index = most work, first
    const int s = blockIdx.z;
    int seg0, len;
    if (!load_segment(prm.cu_seqlens, s, prm.T, prm.max_seqlen, seg0, len, 30)) return;
    if (jt * 128 >= len) return;
    const int G = prm.hq / prm.hkv;

    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t s_base = smem_addr(smem);

    if (tid == 0) {
        mbar_init(bar_kv, 1);
        mbar_init(bar_qdo, 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_do);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_st = tmem;               // S^T   [0, 128)
    const uint32_t t_dpt = tmem + 128;        // dP^T  [128, 256)
    const uint32_t t_dv = tmem + 256;         // dV    [256, 256 + D)
    const uint32_t t_dk = tmem + 256 + D;     // dK    [256 + D, 256 + 2D)
    const uint32_t t_dq = tmem;               // partial dQ reuses S^T's columns
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;

    const int kv_row0 = seg0 + jt * 128;

    KeptTileWalk walk;
    walk.kept_idx = prm.kept_idx;
    walk.kept_cnt = prm.kept_cnt;
    walk.nbmax = prm.nbmax;
    walk.hq = prm.hq;
    walk.G = G;
    walk.g = g;
    walk.s = s;
    walk.block_q = prm.block_q;
    walk.first_block = prm.causal ? (jt * 128) / prm.block_q : 0;
    walk.nb = (len + prm.block_q - 1) / prm.block_q;

    constexpr uint32_t kIdescT = idesc_bf16(128, 128, 0, 0);   // S^T, dP^T
    constexpr uint32_t kIdescKV = idesc_bf16(128, D, 0, 1);     // dV, dK: B (dO, Q) MN-major
    constexpr uint32_t kIdescQ = idesc_bf16(128, D, 1, 1);      // dQ: A (dS) and B (K) MN-major
    const int kv_local = jt * 128 + tid;    // this thread's KV row (S^T/dP^T/dV/dK lane)
    const bool kv_valid = kv_local < len;

    uint32_t ph_qdo = 0, ph_mma = 0;
    bool kv_waited = false, ok = true;
    int n_iter = 0;
    int qdo_pending = 0;   // thread 0: Q/dO loads issued but not yet waited on

    bool more = walk.next(true);
    if (more && tid == 0) {
        mbar_arrive_expect_tx(bar_kv, 2 * L::kTile);
        for (int c = 0; c < L::kPanels; ++c) {
            tma_load_3d(smem + L::kK + c * kPanelBytes, &tm_k, bar_kv, c * 64, g, kv_row0);
            tma_load_3d(smem + L::kV + c * kPanelBytes, &tm_v, bar_kv, c * 64, g, kv_row0);
        }
        mbar_arrive_expect_tx(bar_qdo, 2 * L::kTile);
        ++qdo_pending;
        for (int c = 0; c < L::kPanels; ++c) {
            tma_load_3d(smem + L::kQ + c * kPanelBytes, &tm_q, bar_qdo, c * 64, walk.h, seg0 + walk.tile * 128);
            tma_load_3d(smem + L::kDO + c * kPanelBytes, &tm_do, bar_qdo, c * 64, walk.h, seg0 + walk.tile * 128);
        }
    }

    while (more) {
        const int h = walk.h, qt = walk.tile;
        // per-column (query row) vectors of this tile
        {
            const int q_local = qt * 128 + tid;
            float l2 = 0.f, dd = 0.f, w = 0.f;
            if (q_local < len) {
                const size_t idx = (size_t)h * prm.T + seg0 + q_local;
                l2 = prm.lse[idx] * 1.4426950408889634f;
                dd = prm.Dvec[idx];
                w = prm.block_weight[((size_t)s * prm.hq + h) * prm.nbmax + q_local / prm.block_q];
            }
            lse2_s[tid] = l2;
            dvec_s[tid] = dd;
            w_s[tid] = w;
        }
        if (tid == 0) {
            bool w_ok = kv_waited || mbar_wait(bar_kv, 0, 11);
            kv_waited = w_ok;
            w_ok = w_ok && mbar_wait(bar_qdo, ph_qdo, 12);
            if (w_ok) {
                --qdo_pending;
                ph_qdo ^= 1;
                tc_fence_after();
                const uint32_t ka = s_base + L::kK, va = s_base + L::kV;
                const uint32_t qa = s_base + L::kQ, da = s_base + L::kDO;
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    mma_bf16_ss(t_st, desc_kmajor(ka, k), desc_kmajor(qa, k), kIdescT, k > 0);
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    mma_bf16_ss(t_dpt, desc_kmajor(va, k), desc_kmajor(da, k), kIdescT, k > 0);
                mma_commit(bar_mma);
            } else {
                *abort_flag = 1;
            }
        }
        __syncthreads();
        if (*abort_flag) { ok = false; break; }
        if (!mbar_wait(bar_mma, ph_mma, 13)) *abort_flag = 1;
        ph_mma ^= 1;
        __syncthreads();
        if (*abort_flag) { ok = false; break; }
        tc_fence_after();

        // ---- P^T and dS^T for this thread's KV row ----
        const uint32_t pt_base = s_base + L::kPt, dst_base = s_base + L::kDSt;
        const int q0 = qt * 128;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float sv[32], dpv[32];
            tmem_ld32(t_st + lane_off + c * 32, sv);
            tmem_ld32(t_dpt + lane_off + c * 32, dpv);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t pk[4], dk_[4];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    float pv[2], dsv[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int col = c * 32 + ch * 8 + e2 * 2 + u;
                        const int q_local = q0 + col;
                        const bool valid = kv_valid && q_local < len && (!prm.causal || kv_local <= q_local);
                        const float p = valid ? fast_exp2(sv[ch * 8 + e2 * 2 + u] * prm.scale_log2 - lse2_s[col]) : 0.f;
                        const float w = w_s[col];
                        pv[u] = p * w;
                        dsv[u] = p * (dpv[ch * 8 + e2 * 2 + u] - dvec_s[col]) * w;
                    }
                    pk[e2] = pack_bf16(pv[0], pv[1]);
                    dk_[e2] = pack_bf16(dsv[0], dsv[1]);
                }
                const uint32_t off = sw128_chunk_offset(tid, c * 4 + ch);
                st_shared_v4(pt_base + off, pk[0], pk[1], pk[2], pk[3]);
                st_shared_v4(dst_base + off, dk_[0], dk_[1], dk_[2], dk_[3]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t ka = s_base + L::kK;
            const uint32_t qa = s_base + L::kQ, da = s_base + L::kDO;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16_ss(t_dv, desc_kmajor(pt_base, k), desc_mnmajor(da, k), kIdescKV,
                            (n_iter > 0 || k > 0) ? 1u : 0u);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16_ss(t_dk, desc_kmajor(dst_base, k), desc_mnmajor(qa, k), kIdescKV,
                            (n_iter > 0 || k > 0) ? 1u : 0u);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16_ss(t_dq, desc_mnmajor(dst_base, k), desc_mnmajor(ka, k), kIdescQ, k > 0);
            mma_commit(bar_mma);
        }
        if (!mbar_wait(bar_mma, ph_mma, 14)) *abort_flag = 1;
        ph_mma ^= 1;
        // the walk's next tile: its Q/dO load overlaps the dQ reduction below
        more = walk.next(false);
        __syncthreads();
        if (*abort_flag) { ok = false; break; }
        tc_fence_after();
        if (more && tid == 0) {
            mbar_arrive_expect_tx(bar_qdo, 2 * L::kTile);
            ++qdo_pending;
            for (int c = 0; c < L::kPanels; ++c) {
                tma_load_3d(smem + L::kQ + c * kPanelBytes, &tm_q, bar_qdo, c * 64, walk.h, seg0 + walk.tile * 128);
                tma_load_3d(smem + L::kDO + c * kPanelBytes, &tm_do, bar_qdo, c * 64, walk.h, seg0 + walk.tile * 128);
            }
        }

        // ---- partial dQ of this tile: thread r owns query row r ----
        {
            const int q_local = q0 + tid;
            const bool row_ok = q_local < len && w_s[tid] != 0.f;
            float* dst = prm.dq_acc + ((size_t)(seg0 + q_local) * prm.hq + h) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                float v[32];
                tmem_ld32(t_dq + lane_off + c * 32, v);
                if (row_ok) {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        atomicAdd(reinterpret_cast<float4*>(dst + c * 32 + e * 4),
                                  make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]));
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        ++n_iter;
    }

    if (ok) {
        // ---- epilogue: dV, dK (x softmax_scale) for this thread's KV row ----
        const size_t orow = ((size_t)(kv_row0 + tid) * prm.hkv + g) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            float v[32], k[32];
            if (n_iter > 0) {
                tmem_ld32(t_dv + lane_off + c * 32, v);
                tmem_ld32(t_dk + lane_off + c * 32, k);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) { v[e] = 0.f; k[e] = 0.f; }
            }
            if (kv_valid) {
#pragma unroll
                for (int e8 = 0; e8 < 4; ++e8) {
                    uint4 pv, pk;
                    pv.x = pack_bf16(v[e8 * 8 + 0], v[e8 * 8 + 1]);
                    pv.y = pack_bf16(v[e8 * 8 + 2], v[e8 * 8 + 3]);
                    pv.z = pack_bf16(v[e8 * 8 + 4], v[e8 * 8 + 5]);
                    pv.w = pack_bf16(v[e8 * 8 + 6], v[e8 * 8 + 7]);
                    pk.x = pack_bf16(k[e8 * 8 + 0] * prm.scale, k[e8 * 8 + 1] * prm.scale);
                    pk.y = pack_bf16(k[e8 * 8 + 2] * prm.scale, k[e8 * 8 + 3] * prm.scale);
                    pk.z = pack_bf16(k[e8 * 8 + 4] * prm.scale, k[e8 * 8 + 5] * prm.scale);
                    pk.w = pack_bf16(k[e8 * 8 + 6] * prm.scale, k[e8 * 8 + 7] * prm.scale);
                    *reinterpret_cast<uint4*>(prm.dv + orow + c * 32 + e8 * 8) = pv;
                    *reinterpret_cast<uint4*>(prm.dk + orow + c * 32 + e8 * 8) = pk;
                }
            }
        }
    } else if (tid == 0) {
        // a wait gave up: let this CTA's own TMA copies land (bounded) before exit
        if (!kv_waited && n_iter == 0) mbar_wait(bar_kv, 0, 15);
        while (qdo_pending > 0 && mbar_wait(bar_qdo, ph_qdo, 15)) { --qdo_pending; ph_qdo ^= 1; }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace lf
