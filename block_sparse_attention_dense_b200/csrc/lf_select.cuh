// LazyFlash selection on the GPU (article section "Un budget sur la masse de
// gradient, et un tirage qui garde le gradient non biaisé"):
//   1. norms_rowdot_kernel: ||dO_b||_F per (segment, head, block) and
//      D[h][t] = <dO_t, O_t>, in one streaming pass over dO and O;
//   2. select_kernel: per (segment, head) the budgeted threshold tau by
//      bisection, the Philox keep draw, the 1/p weights and the ascending
//      kept-block list;
//   3. dq_convert_kernel: fp32 dQ accumulator -> scaled bf16 dQ.
#pragma once

#include "lf_device.cuh"

namespace lf {

// ---------------------------------------------------------------------------
// 1. Block norms and D.  One CTA of 4 warps per (block, head, segment).  Each
// warp walks rows of the block; a lane owns d/32 consecutive elements of a
// row.  Sums of squares and dot products accumulate in fp32.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) norms_rowdot_kernel(
    const int32_t* __restrict__ cu_seqlens, int T, int max_seqlen, int hq, int block, int nbmax,
    const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ o,
    float* __restrict__ norms, float* __restrict__ Dout, int write_norms) {
    constexpr int EPL = D / 32;   // elements per lane: 2 or 4
    const int i = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    int seg0, len;
    if (!load_segment(cu_seqlens, s, T, max_seqlen, seg0, len, 40)) return;
    const int seg1 = seg0 + len;
    const int nb = (len + block - 1) / block;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ float red[4];
    if (i >= nb) {
        // blocks past the segment's end carry zero norm
        if (write_norms && i < nbmax && threadIdx.x == 0)
            norms[((size_t)s * hq + h) * nbmax + i] = 0.f;
        return;
    }
    const int r0 = seg0 + i * block;
    const int r1 = min(r0 + block, seg1);
    float ss = 0.f;
    for (int t = r0 + warp; t < r1; t += 4) {
        const size_t base = ((size_t)t * hq + h) * D + lane * EPL;
        float a[EPL], b[EPL];
        if constexpr (EPL == 4) {
            uint2 ua = *reinterpret_cast<const uint2*>(dout + base);
            uint2 ub = *reinterpret_cast<const uint2*>(o + base);
            const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&ua);
            const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&ub);
            float2 a0 = __bfloat1622float2(pa[0]), a1 = __bfloat1622float2(pa[1]);
            float2 b0 = __bfloat1622float2(pb[0]), b1 = __bfloat1622float2(pb[1]);
            a[0] = a0.x; a[1] = a0.y; a[2] = a1.x; a[3] = a1.y;
            b[0] = b0.x; b[1] = b0.y; b[2] = b1.x; b[3] = b1.y;
        } else {
            uint32_t ua = *reinterpret_cast<const uint32_t*>(dout + base);
            uint32_t ub = *reinterpret_cast<const uint32_t*>(o + base);
            float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ua));
            float2 b0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ub));
            a[0] = a0.x; a[1] = a0.y;
            b[0] = b0.x; b[1] = b0.y;
        }
        float dsq = 0.f, dot = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            dsq = fmaf(a[e], a[e], dsq);
            dot = fmaf(a[e], b[e], dot);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        if (lane == 0) Dout[(size_t)h * T + t] = dot;
        ss += dsq;
    }
    if (!write_norms) return;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (threadIdx.x == 0)
        norms[((size_t)s * hq + h) * nbmax + i] = sqrtf((red[0] + red[1]) + (red[2] + red[3]));
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): ten rounds of two 32x32
// multiplies whose high halves are xored into the other two words together
// with the round key; the key advances by the golden-ratio Weyl constants.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t lo_a = 0xD2511F53u * c.x, hi_a = __umulhi(0xD2511F53u, c.x);
        const uint32_t lo_b = 0xCD9E8D57u * c.z, hi_b = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi_b ^ c.y ^ k.x, lo_b, hi_a ^ c.w ^ k.y, lo_a);
        k.x += 0x9E3779B9u;
        k.y += 0xBB67AE85u;
    }
    return c;
}

// fp64 sum in the fixed order the selection pins: lane l accumulates its
// strided elements in index order, then five xor-butterfly rounds.  Every
// operation is an explicitly rounded fp64 add (no contraction).
__device__ __forceinline__ double warp_butterfly_sum(double v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

// ---------------------------------------------------------------------------
// 2. One warp per (segment, head).  Shared memory holds the head's norms as
// fp64 (nbmax entries).  RULE 0: the LazyFlash budget (param = delta): tau is
// the largest threshold whose expected discarded mass sum (1 - p) m stays
// within delta * sum m.  RULE 1: fixed fraction (param = f): tau is the
// largest threshold whose expected kept count sum p reaches f * n.  Both draw
// keep ~ Bernoulli(p = min(1, m/tau)) from Philox and weight kept blocks 1/p.
// RULE 2: top-k (k = ceil(f * n)): the k largest norms, weight 1, no draw.
// ---------------------------------------------------------------------------
template <int RULE>
__global__ void __launch_bounds__(32) select_kernel(
    const int32_t* __restrict__ cu_seqlens, int T, int max_seqlen, int hq, int block, int nbmax,
    const float* __restrict__ norms, double param, uint64_t seed, uint64_t step,
    double* __restrict__ tau_out, float* __restrict__ w_out, uint8_t* __restrict__ keep_out,
    int32_t* __restrict__ kept_idx, int32_t* __restrict__ kept_cnt) {
    extern __shared__ double m_s[];
    const int h = blockIdx.x, s = blockIdx.y, lane = threadIdx.x;
    int seg0, len;
    if (!load_segment(cu_seqlens, s, T, max_seqlen, seg0, len, 41)) return;
    const int n = (len + block - 1) / block;
    if (n > nbmax) {   // cannot happen when len <= max_seqlen; keeps the smem walk in bounds
        if (lane == 0) report_error(42, kErrBadSegments);
        return;
    }
    const size_t base = ((size_t)s * hq + h) * nbmax;
    for (int i = lane; i < n; i += 32) m_s[i] = static_cast<double>(norms[base + i]);
    __syncwarp();

    double total = 0.0, mx = 0.0;
    for (int i = lane; i < n; i += 32) {
        total = __dadd_rn(total, m_s[i]);
        mx = fmax(mx, m_s[i]);
    }
    total = warp_butterfly_sum(total);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));

    double tau = 0.0;
    int k_top = 0;
    if (RULE == 0 && param > 0.0 && total > 0.0) {
        const double budget = __dmul_rn(param, total);
        double lo = 0.0, hi = __ddiv_rn(mx, __dsub_rn(1.0, param));
        for (int it = 0; it < 64; ++it) {
            const double mid = __dmul_rn(0.5, __dadd_rn(lo, hi));
            double f = 0.0;
            for (int i = lane; i < n; i += 32) {
                const double m = m_s[i];
                const double t = (m >= mid) ? 0.0 : __dmul_rn(__dsub_rn(1.0, __ddiv_rn(m, mid)), m);
                f = __dadd_rn(f, t);
            }
            f = warp_butterfly_sum(f);
            if (f <= budget) lo = mid; else hi = mid;
        }
        tau = lo;
    } else if (RULE == 1 && n > 0 && total > 0.0 && param < 1.0) {
        const double target = __dmul_rn(param, static_cast<double>(n));
        double lo = 0.0, hi = __ddiv_rn(total, target);
        for (int it = 0; it < 64; ++it) {
            const double mid = __dmul_rn(0.5, __dadd_rn(lo, hi));
            double g = 0.0;
            for (int i = lane; i < n; i += 32) {
                const double m = m_s[i];
                g = __dadd_rn(g, (m >= mid) ? 1.0 : __ddiv_rn(m, mid));
            }
            g = warp_butterfly_sum(g);
            if (g >= target) lo = mid; else hi = mid;
        }
        tau = lo;
    } else if (RULE == 2) {
        k_top = min(n, static_cast<int>(ceil(__dmul_rn(param, static_cast<double>(n)))));
    }

    const uint2 key = make_uint2(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
    int count = 0;
    for (int i0 = 0; i0 < nbmax; i0 += 32) {
        const int i = i0 + lane;
        bool kept = false;
        float w = 0.f;
        if (i < n) {
            if (RULE == 2) {
                // rank = blocks with a larger norm, or an equal norm and a lower index
                const double mi = m_s[i];
                int rank = 0;
                for (int j = 0; j < n; ++j) {
                    const double mj = m_s[j];
                    rank += (mj > mi || (mj == mi && j < i)) ? 1 : 0;
                }
                kept = rank < k_top;
                if (rank == k_top - 1) tau = mi;
                w = kept ? 1.f : 0.f;
            } else {
                double p = 1.0;
                if (tau != 0.0) p = fmin(1.0, __ddiv_rn(m_s[i], tau));
                if (p >= 1.0) {
                    kept = true;
                } else {
                    const uint4 r = philox4x32_10(
                        make_uint4(static_cast<uint32_t>(i), static_cast<uint32_t>(h),
                                   static_cast<uint32_t>(s), static_cast<uint32_t>(step)),
                        key);
                    kept = static_cast<double>(r.x >> 8) < __dmul_rn(p, 16777216.0);
                }
                if (kept) w = __double2float_rn(__ddiv_rn(1.0, p));
            }
        }
        if (i < nbmax) {
            keep_out[base + i] = kept ? 1 : 0;
            w_out[base + i] = w;
        }
        const uint32_t ballot = __ballot_sync(0xffffffffu, kept);
        if (kept) kept_idx[base + count + __popc(ballot & ((1u << lane) - 1u))] = i;
        count += __popc(ballot);
    }
    for (int i = count + lane; i < nbmax; i += 32) kept_idx[base + i] = -1;
    if (RULE == 2) {
        // the lane that held the k-th largest norm owns tau
        const uint32_t holder = __ballot_sync(0xffffffffu, tau != 0.0);
        if (holder) tau = __shfl_sync(0xffffffffu, tau, __ffs(holder) - 1);
    }
    if (lane == 0) {
        tau_out[(size_t)s * hq + h] = tau;
        kept_cnt[(size_t)s * hq + h] = count;
    }
}

// ---------------------------------------------------------------------------
// 3. dK, dV = scale * accumulator, rounded to bf16 (8 elements per thread).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dq_convert_kernel(const float4* __restrict__ acc,
                                                         uint4* __restrict__ dq, size_t n8,
                                                         float scale) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8;
         i += (size_t)gridDim.x * blockDim.x) {
        const float4 a = acc[2 * i], b = acc[2 * i + 1];
        uint4 r;
        r.x = pack_bf16(a.x * scale, a.y * scale);
        r.y = pack_bf16(a.z * scale, a.w * scale);
        r.z = pack_bf16(b.x * scale, b.y * scale);
        r.w = pack_bf16(b.z * scale, b.w * scale);
        dq[i] = r;
    }
}

// ---------------------------------------------------------------------------
// 4. The dQ accumulator, kept blocks only.
// ---------------------------------------------------------------------------
// The backward adds into the fp32 dQ accumulator only the rows of blocks whose
// weight is non-zero (dropped blocks contribute exactly nothing), so only those rows
// are zeroed beforehand and read afterwards; the bf16 dQ rows of the other blocks are
// written as zeros.  One CTA per (block, head, segment); accumulator head-major
// [H][T][D] fp32, output [T][H][D] bf16.
__global__ void __launch_bounds__(256) dq_acc_zero_kept_kernel(const int32_t* __restrict__ cu_seqlens, int T,
                                                               int max_seqlen, int H, int D, int block_q,
                                                               int nbmax, const float* __restrict__ w,
                                                               float* __restrict__ acc) {
    const int b = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    int seg0, len;
    if (!load_segment(cu_seqlens, s, T, max_seqlen, seg0, len, 50)) return;
    if (b * block_q >= len || w[((size_t)s * H + h) * nbmax + b] == 0.f) return;
    const int r0 = b * block_q, r1 = min(len, r0 + block_q);
    float4* dst = reinterpret_cast<float4*>(acc + ((size_t)h * T + seg0 + r0) * D);
    const int n4 = (r1 - r0) * D / 4;
    for (int i = threadIdx.x; i < n4; i += blockDim.x) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

template <int D>
__global__ void __launch_bounds__(256) dq_acc_to_thd_kept_kernel(const int32_t* __restrict__ cu_seqlens, int T,
                                                                 int max_seqlen, int H, int block_q, int nbmax,
                                                                 const float* __restrict__ w,
                                                                 const float* __restrict__ acc,
                                                                 uint4* __restrict__ out, float scale) {
    const int b = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    int seg0, len;
    if (!load_segment(cu_seqlens, s, T, max_seqlen, seg0, len, 51)) return;
    if (b * block_q >= len) return;
    const bool kept = w[((size_t)s * H + h) * nbmax + b] != 0.f;
    const int r0 = b * block_q, r1 = min(len, r0 + block_q);
    constexpr int d8 = D / 8;
    const int n = (r1 - r0) * d8;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int c = i % d8;
        const size_t t = (size_t)seg0 + r0 + i / d8;
        uint4 r = make_uint4(0u, 0u, 0u, 0u);
        if (kept) {
            const float4* src = reinterpret_cast<const float4*>(acc + ((size_t)h * T + t) * D + c * 8);
            const float4 a = src[0], bb = src[1];
            r.x = pack_bf16(a.x * scale, a.y * scale);
            r.y = pack_bf16(a.z * scale, a.w * scale);
            r.z = pack_bf16(bb.x * scale, bb.y * scale);
            r.w = pack_bf16(bb.z * scale, bb.w * scale);
        }
        out[(t * H + h) * d8 + c] = r;
    }
}

}  // namespace lf
