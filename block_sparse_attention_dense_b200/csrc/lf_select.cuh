// LazyFlash selection on the GPU (article section "Un budget sur la masse de
// gradient, et un tirage qui garde le gradient non biaisé"):
//   1. norms_rowdot_kernel: ||dO_b||_F per (segment, head, block) and, when
//      asked, D[h][t] = <dO_t, O_t>, in one streaming pass over dO (and O);
//   2. select_kernel: per (segment, head) the budgeted threshold tau by
//      bisection, the Philox keep draw, the 1/p weights and the ascending
//      kept-block list;
//   3. dq_convert_kernel: fp32 accumulator -> scaled bf16;
//   4. the backward's prologue over kept blocks (dQ accumulator rows zeroed,
//      D computed when the caller did not pass it) and the dQ conversion.
#pragma once

#include "lf_device.cuh"

namespace lf {

// ---------------------------------------------------------------------------
// 1. Block norms and D.  One CTA of 8 warps per (block, head, segment).  A lane
// loads 16 bytes (8 bf16) of a row, so a warp instruction covers 32 / (d / 8)
// rows, and each warp keeps four such loads per tensor in flight.  Sums of
// squares and dot products accumulate in fp32.  Without D (Dout == nullptr)
// only dO is read.
// ---------------------------------------------------------------------------
constexpr int kNormThreads = 256;

template <int D>
__device__ __forceinline__ float bf16x8_dot(uint4 a, uint4 b) {
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(pa[e]), y = __bfloat1622float2(pb[e]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
    }
    return acc;
}

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Rows [r0, r1) of head h: returns this thread's sum of squares of dO; writes
// D[h][t] = <dO_t, O_t> when Dout is given.  Every thread of the CTA calls it.
template <int D>
__device__ __forceinline__ float block_rows_pass(int r0, int r1, int h, int hq, int T,
                                                 const __nv_bfloat16* __restrict__ dout,
                                                 const __nv_bfloat16* __restrict__ o,
                                                 float* __restrict__ Dout) {
    constexpr int LPR = D / 8;                  // lanes per row
    constexpr int RPW = 32 / LPR;               // rows per warp instruction
    constexpr int STEP = (kNormThreads / 32) * RPW;
    constexpr int U = 4;                        // loads in flight per tensor and thread
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR, c8 = (lane % LPR) * 8;
    float ss = 0.f;
    for (int t0 = r0 + warp * RPW + sub; t0 < r1 + sub; t0 += STEP * U) {
        uint4 a[U], b[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = t0 + u * STEP;
            a[u] = b[u] = make_uint4(0u, 0u, 0u, 0u);
            if (t < r1) {
                const size_t off = ((size_t)t * hq + h) * D + c8;
                a[u] = ld_stream16(dout + off);
                if (Dout) b[u] = ld_stream16(o + off);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            ss += bf16x8_dot<D>(a[u], a[u]);
            if (Dout) {
                float dot = bf16x8_dot<D>(a[u], b[u]);
#pragma unroll
                for (int off = LPR / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
                const int t = t0 + u * STEP;
                if (lane % LPR == 0 && t < r1) Dout[(size_t)h * T + t] = dot;
            }
        }
    }
    return ss;
}

template <int D>
__global__ void __launch_bounds__(kNormThreads) norms_rowdot_kernel(
    const int32_t* __restrict__ cu_seqlens, int T, int max_seqlen, int hq, int block, int nbmax,
    const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ o,
    float* __restrict__ norms, float* __restrict__ Dout, int write_norms) {
    const int i = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    int seg0, len;
    if (!load_segment(cu_seqlens, s, T, max_seqlen, seg0, len, 40)) return;
    const int nb = (len + block - 1) / block;
    __shared__ float red[kNormThreads / 32];
    if (i >= nb) {
        // blocks past the segment's end carry zero norm
        if (write_norms && i < nbmax && threadIdx.x == 0)
            norms[((size_t)s * hq + h) * nbmax + i] = 0.f;
        return;
    }
    const int r0 = seg0 + i * block;
    const int r1 = min(r0 + block, seg0 + len);
    float ss = block_rows_pass<D>(r0, r1, h, hq, T, dout, o, Dout);
    if (!write_norms) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < kNormThreads / 32; ++w) t += red[w];
        norms[((size_t)s * hq + h) * nbmax + i] = sqrtf(t);
    }
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
// 2. Selection: one CTA of 8 warps per (segment, head).  Shared memory holds the
// head's norms (fp32, nbmax entries; converted to fp64 exactly where used).
// RULE 0: the LazyFlash budget (param = delta): tau is the largest threshold
// whose expected discarded mass sum (1 - p) m stays within delta * sum m.
// RULE 1: fixed fraction (param = f): tau is the largest threshold whose
// expected kept count sum p reaches f * n.  Both draw keep ~ Bernoulli(p =
// min(1, m/tau)) from Philox and weight kept blocks 1/p.  RULE 2: top-k (k =
// ceil(f * n)): the k largest norms (ties to the lower index), weight 1, no draw.
//
// The 64 bisection steps are taken four at a time: the fifteen midpoints the
// next four steps can visit (a depth-4 tree below the current bracket, each
// computed by the same fp64 operations the sequential steps would use) are
// evaluated at once, two per warp, every evaluation in the pinned summation
// order; the steps then follow the tree.  The result is the sequential
// bisection's, bit for bit.
// ---------------------------------------------------------------------------
constexpr int kSelectThreads = 256;

// One block's term of the bisection's test at threshold t = mid, the test
// multiplied through by t so that it takes no division.  RULE 0: the discarded
// mass (1 - m/t) m becomes m t - m^2 (one fused multiply-add; the square of an
// fp32 norm is exact in fp64), 0 for m >= t.  RULE 1: the keep probability
// min(1, m/t) becomes min(t, m), exact.
template <int RULE>
__device__ __forceinline__ double select_term(float mf, double mid) {
    const double m = static_cast<double>(mf);
    if (RULE == 0) return (m >= mid) ? 0.0 : __fma_rn(m, mid, -__dmul_rn(m, m));
    return (m >= mid) ? mid : m;
}

// sum_i term(m_i, mid) in the pinned order (lane l: i = l, l + 32, ... in index
// order, then the butterfly); the whole warp calls it and every lane gets it.
template <int RULE>
__device__ __forceinline__ double pinned_eval(const float* m_s, int n, double mid) {
    const int lane = threadIdx.x & 31;
    double acc = 0.0;
    int i = lane;
    for (; i + 96 < n; i += 128) {   // four independent terms in flight, adds in order
        const double t0 = select_term<RULE>(m_s[i], mid), t1 = select_term<RULE>(m_s[i + 32], mid);
        const double t2 = select_term<RULE>(m_s[i + 64], mid), t3 = select_term<RULE>(m_s[i + 96], mid);
        acc = __dadd_rn(acc, t0);
        acc = __dadd_rn(acc, t1);
        acc = __dadd_rn(acc, t2);
        acc = __dadd_rn(acc, t3);
    }
    for (; i < n; i += 32) acc = __dadd_rn(acc, select_term<RULE>(m_s[i], mid));
    return warp_butterfly_sum(acc);
}

// The same sums at two thresholds at once (two independent chains, each in the
// pinned order).
template <int RULE>
__device__ __forceinline__ void pinned_eval2(const float* m_s, int n, double t0, double t1,
                                             double& v0, double& v1) {
    const int lane = threadIdx.x & 31;
    double a0 = 0.0, a1 = 0.0;
    int i = lane;
    for (; i + 32 < n; i += 64) {
        const float m0 = m_s[i], m1 = m_s[i + 32];
        const double p0 = select_term<RULE>(m0, t0), q0 = select_term<RULE>(m0, t1);
        const double p1 = select_term<RULE>(m1, t0), q1 = select_term<RULE>(m1, t1);
        a0 = __dadd_rn(a0, p0);
        a1 = __dadd_rn(a1, q0);
        a0 = __dadd_rn(a0, p1);
        a1 = __dadd_rn(a1, q1);
    }
    for (; i < n; i += 32) {
        const float m0 = m_s[i];
        a0 = __dadd_rn(a0, select_term<RULE>(m0, t0));
        a1 = __dadd_rn(a1, select_term<RULE>(m0, t1));
    }
    v0 = warp_butterfly_sum(a0);
    v1 = warp_butterfly_sum(a1);
}

__device__ __forceinline__ double bisect_mid(double lo, double hi) {
    return __dmul_rn(0.5, __dadd_rn(lo, hi));
}

template <int RULE>
__global__ void __launch_bounds__(kSelectThreads) select_kernel(
    const int32_t* __restrict__ cu_seqlens, int T, int max_seqlen, int hq, int block, int nbmax,
    const float* __restrict__ norms, double param, uint64_t seed, uint64_t step,
    double* __restrict__ tau_out, float* __restrict__ w_out, uint8_t* __restrict__ keep_out,
    int32_t* __restrict__ kept_idx, int32_t* __restrict__ kept_cnt) {
    extern __shared__ float m_s[];
    __shared__ double red_s[2];
    __shared__ int flag_s[16];
    __shared__ int wcnt_s[2][kSelectThreads / 32];
    __shared__ uint32_t hist_s[256];
    __shared__ uint32_t radix_s[2];
    const int h = blockIdx.x, s = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int seg0, len;
    if (!load_segment(cu_seqlens, s, T, max_seqlen, seg0, len, 41)) return;
    const int n = (len + block - 1) / block;
    if (n > nbmax) {   // cannot happen when len <= max_seqlen; keeps the smem walk in bounds
        if (tid == 0) report_error(42, kErrBadSegments);
        return;
    }
    const size_t base = ((size_t)s * hq + h) * nbmax;
    for (int i = tid; i < n; i += kSelectThreads) m_s[i] = norms[base + i];
    __syncthreads();

    // total mass in the pinned order, and the largest norm
    if (warp == 0) {
        double total = 0.0, mx = 0.0;
        for (int i = lane; i < n; i += 32) {
            total = __dadd_rn(total, static_cast<double>(m_s[i]));
            mx = fmax(mx, static_cast<double>(m_s[i]));
        }
        total = warp_butterfly_sum(total);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) {
            red_s[0] = total;
            red_s[1] = mx;
        }
    }
    __syncthreads();
    const double total = red_s[0], mx = red_s[1];

    double tau = 0.0;
    uint32_t kth_key = 0;   // top-k: bit pattern of the k-th largest norm
    int k_top = 0, eq_keep = 0;
    const bool bisect = (RULE == 0 && param > 0.0 && total > 0.0) ||
                        (RULE == 1 && n > 0 && total > 0.0 && param < 1.0);
    if (bisect) {
        // RULE 0: feasible iff f(mid) <= delta * M; RULE 1: iff g(mid) >= f * n; both
        // evaluated multiplied through by mid (sum of the terms above against crit * mid)
        const double crit = RULE == 0 ? __dmul_rn(param, total) : __dmul_rn(param, static_cast<double>(n));
        double lo = 0.0, hi = RULE == 0 ? __ddiv_rn(mx, __dsub_rn(1.0, param)) : __ddiv_rn(total, crit);
        // heap node j of the tree below (lo, hi): bit 1 of the path = the step moved lo
        // up to its midpoint, bit 0 = hi down; the midpoint is formed by the same
        // operations the sequential steps would take
        auto node_mid = [&](int node) {
            const int depth = 31 - __clz(node);
            double l = lo, u = hi;
            for (int bit = depth - 1; bit >= 0; --bit) {
                const double mid = bisect_mid(l, u);
                if ((node >> bit) & 1) l = mid; else u = mid;
            }
            return bisect_mid(l, u);
        };
        auto feasible = [&](double v, double t) {
            const double rhs = __dmul_rn(crit, t);
            return RULE == 0 ? (v <= rhs) : (v >= rhs);
        };
        for (int it = 0; it < 64;) {
            // four steps per round: the fifteen nodes of a depth-4 tree, nodes warp + 1
            // and warp + 9 per warp (64 = 16 rounds of 4)
            const int levels = min(4, 64 - it);
            const int nodes = (1 << levels) - 1;
            const int n0 = warp + 1, n1 = warp + 9;
            if (n0 <= nodes) {
                const double t0 = node_mid(n0);
                if (n1 <= nodes) {
                    const double t1 = node_mid(n1);
                    double v0, v1;
                    pinned_eval2<RULE>(m_s, n, t0, t1, v0, v1);
                    if (lane == 0) {
                        flag_s[n0 - 1] = feasible(v0, t0);
                        flag_s[n1 - 1] = feasible(v1, t1);
                    }
                } else {
                    const double v0 = pinned_eval<RULE>(m_s, n, t0);
                    if (lane == 0) flag_s[n0 - 1] = feasible(v0, t0);
                }
            }
            __syncthreads();
            int node = 1;
            for (int d = 0; d < levels; ++d) {
                const double mid = bisect_mid(lo, hi);
                if (flag_s[node - 1]) {
                    lo = mid;
                    node = 2 * node + 1;
                } else {
                    hi = mid;
                    node = 2 * node;
                }
            }
            it += levels;
            __syncthreads();   // flag_s is rewritten by the next round
        }
        tau = lo;
    } else if (RULE == 2) {
        k_top = min(n, static_cast<int>(ceil(__dmul_rn(param, static_cast<double>(n)))));
        if (k_top > 0) {
            // radix select of the k-th largest norm: norms are >= 0, so their fp32 bit
            // patterns order like their values; one byte per round, most significant first
            uint32_t prefix = 0;
            int kr = k_top;
            for (int shift = 24; shift >= 0; shift -= 8) {
                hist_s[tid] = 0;
                __syncthreads();
                const uint32_t hi_mask = shift == 24 ? 0u : (0xffffffffu << (shift + 8));
                for (int i = tid; i < n; i += kSelectThreads) {
                    const uint32_t key = __float_as_uint(m_s[i]);
                    if ((key & hi_mask) == (prefix & hi_mask)) atomicAdd(&hist_s[(key >> shift) & 255u], 1u);
                }
                __syncthreads();
                if (tid == 0) {
                    int acc = 0, bin = 255;
                    for (; bin > 0; --bin) {
                        if (acc + static_cast<int>(hist_s[bin]) >= kr) break;
                        acc += static_cast<int>(hist_s[bin]);
                    }
                    radix_s[0] = prefix | (static_cast<uint32_t>(bin) << shift);
                    radix_s[1] = static_cast<uint32_t>(kr - acc);
                }
                __syncthreads();
                prefix = radix_s[0];
                kr = static_cast<int>(radix_s[1]);
                __syncthreads();
            }
            kth_key = prefix;
            eq_keep = kr;   // blocks equal to the k-th largest kept, lowest indices first
            tau = static_cast<double>(__uint_as_float(kth_key));
        }
    }

    // draw, weights and the ascending kept list, 256 blocks per round
    const uint2 key = make_uint2(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
    const uint32_t lt_mask = (1u << lane) - 1u;
    int count = 0, eq_seen = 0;
    for (int c0 = 0; c0 < nbmax; c0 += kSelectThreads) {
        const int i = c0 + tid;
        bool kept = false;
        float w = 0.f;
        if (RULE == 2) {
            // ties at the k-th largest norm go to the lower indices: count the equal
            // ones before this block (an ordered scan over the CTA)
            const uint32_t mk = i < n ? __float_as_uint(m_s[i]) : 0u;
            const bool eq = k_top > 0 && i < n && mk == kth_key;
            const uint32_t eb = __ballot_sync(0xffffffffu, eq);
            if (lane == 0) wcnt_s[0][warp] = __popc(eb);
            __syncthreads();
            int before = eq_seen, round_total = 0;
#pragma unroll
            for (int q = 0; q < kSelectThreads / 32; ++q) {
                const int c = wcnt_s[0][q];
                if (q < warp) before += c;
                round_total += c;
            }
            before += __popc(eb & lt_mask);
            eq_seen += round_total;
            kept = k_top > 0 && i < n && (mk > kth_key || (eq && before < eq_keep));
            w = kept ? 1.f : 0.f;
        } else if (i < n) {
            double p = 1.0;
            if (tau != 0.0) p = fmin(1.0, __ddiv_rn(static_cast<double>(m_s[i]), tau));
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
        if (i < nbmax) {
            keep_out[base + i] = kept ? 1 : 0;
            w_out[base + i] = w;
        }
        const uint32_t kb = __ballot_sync(0xffffffffu, kept);
        if (lane == 0) wcnt_s[1][warp] = __popc(kb);
        __syncthreads();
        int before = count, round_total = 0;
#pragma unroll
        for (int q = 0; q < kSelectThreads / 32; ++q) {
            const int c = wcnt_s[1][q];
            if (q < warp) before += c;
            round_total += c;
        }
        if (kept) kept_idx[base + before + __popc(kb & lt_mask)] = i;
        count += round_total;
        __syncthreads();   // wcnt_s is rewritten by the next round
    }
    for (int i = count + tid; i < nbmax; i += kSelectThreads) kept_idx[base + i] = -1;
    if (tid == 0) {
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
//
// Prologue: zero the kept blocks' accumulator rows and, when Dw is given (the caller
// passed no D), compute D = <dO_t, O_t> for the kept blocks' rows and write 0 for the
// dropped blocks' rows (the backward reads them, with weight 0, when a 128-row tile
// holds one kept and one dropped 64-row block).
template <int D>
__global__ void __launch_bounds__(kNormThreads) bwd_prologue_kernel(
    const int32_t* __restrict__ cu_seqlens, int T, int max_seqlen, int H, int block_q, int nbmax,
    const float* __restrict__ w, float* __restrict__ acc, const __nv_bfloat16* __restrict__ dout,
    const __nv_bfloat16* __restrict__ o, float* __restrict__ Dw) {
    const int b = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    int seg0, len;
    if (!load_segment(cu_seqlens, s, T, max_seqlen, seg0, len, 50)) return;
    if (b * block_q >= len) return;
    const bool kept = w[((size_t)s * H + h) * nbmax + b] != 0.f;
    const int r0 = b * block_q, r1 = min(len, r0 + block_q);
    if (kept) {
        float4* dst = reinterpret_cast<float4*>(acc + ((size_t)h * T + seg0 + r0) * D);
        const int n4 = (r1 - r0) * D / 4;
        for (int i = threadIdx.x; i < n4; i += blockDim.x) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (Dw) {
        if (kept) {
            (void)block_rows_pass<D>(seg0 + r0, seg0 + r1, h, H, T, dout, o, Dw);
        } else {
            for (int t = seg0 + r0 + threadIdx.x; t < seg0 + r1; t += blockDim.x) Dw[(size_t)h * T + t] = 0.f;
        }
    }
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
