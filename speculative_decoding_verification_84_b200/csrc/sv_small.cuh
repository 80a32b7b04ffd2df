// sv_small.cuh -- short rows (V <= kSmallMaxV): groups of G lanes verify one
// sequence each, from start to end, with the rows in registers.
//
// G (8, 16 or 32) is the smallest group with G >= gamma and 8*G >= V, so a warp
// carries 32/G sequences through the same instructions (c5, V = 64, gamma = 4:
// four sequences per warp, 8 lanes x 8 fp32 each).  Lane l of a group owns
// tokens [l*E, l*E + E) of every row.  The group loads a batch of rows at once
// (every load in flight), then per row: the maximum and the sum of
// 2^(l*k - ceil(max*k_hi)) by shuffles inside the group (the arithmetic of the
// other paths, with the row's exact maximum as offset), or the first argmax when
// T = 0; the accept test's logit l[x_j] comes from the owning lane by one
// shuffle.  Lane j of a group keeps what position j needs, so the log-space test
// of every position [FlashSpec, Metodologia 1] runs in parallel across lanes and
// the first rejection comes from one ballot.  The draw re-reads its one or two
// rows (from L1), forms max(0, p_n - q_n) or p_gamma [Speculative Speculative
// Decoding, Metodologia 2; Desafios 2, "Amostragem Saguaro"], and finds the token
// by an fp64 scan of the lanes' sums inside the group, then inside the lane that
// crosses u * S.  No workspace, no second kernel.
//
// Every lane of a warp runs the same instructions whatever its group's sequence
// needs (rows a group does not read are predicated off); where groups must take
// different branches (greedy or not), the shuffles inside use the mask of the
// lanes that took the branch, and xor offsets below G never leave the group.
#pragma once

#include "sv_common.cuh"

namespace sv {

constexpr int kSmallMaxV = 256;  // rows of at most this many elements take this path
constexpr int kSmallRegs = 4;    // row values per lane held at once (a batch of rows)

template <int G>
__device__ __forceinline__ unsigned group_bits(unsigned ballot)
{
    const int lane = threadIdx.x & 31;
    const unsigned gmask = G == 32 ? 0xffffffffu : ((1u << G) - 1u);
    return (ballot >> (lane & ~(G - 1))) & gmask;
}

template <int ESZ, int G, int E>
__device__ __forceinline__ void small_load_row(const TailArgs& a, int b, int r, bool need, float (&x)[E])
{
    const int gl = threadIdx.x & (G - 1);
    const size_t V = (size_t)a.V;
    if (!need) {
#pragma unroll
        for (int e = 0; e < E; ++e) x[e] = -INFINITY;
        return;
    }
    const unsigned char* base =
        r <= a.gamma ? static_cast<const unsigned char*>(a.tgt) + ((size_t)b * (a.gamma + 1) + r) * V * ESZ
                     : static_cast<const unsigned char*>(a.dft) + ((size_t)b * a.gamma + (r - a.gamma - 1)) * V * ESZ;
    constexpr int kVecElems = 16 / ESZ;
    if (E % kVecElems == 0 && a.V % E == 0) {
        // the lane's E elements are whole 16-byte vectors: rows start 16-byte aligned
        // (checked on the host) and E * ESZ divides the row length
        if (gl * E < a.V) {
#pragma unroll
            for (int k = 0; k < E / kVecElems; ++k) {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + ((size_t)gl * E + k * kVecElems) * ESZ));
                float f[kVecElems];
                unpack<ESZ>(v, f);
#pragma unroll
                for (int e = 0; e < kVecElems; ++e) x[k * kVecElems + e] = f[e];
            }
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) x[e] = -INFINITY;
        }
        return;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int v = gl * E + e;
        x[e] = v < a.V ? load_logit<ESZ>(base, (size_t)v) : -INFINITY;
    }
}

template <int E>
__device__ __forceinline__ float select_e(const float (&x)[E], int e)
{
    float v = x[0];
#pragma unroll
    for (int k = 1; k < E; ++k)
        if (k == e) v = x[k];
    return v;
}

// One row's fold for every group of the warp: softmax groups get (mk, s), mk =
// ceil(max * k_hi) and s the group's fp32 sum of 2^(l*k - mk); greedy groups get
// the first argmax.  `greedy` is uniform within a group.
template <int G, int E>
__device__ __forceinline__ void small_fold(const float (&x)[E], bool greedy, float khi, float klo, float& mk,
                                           float& s, int& arg, int& bad)
{
    const int gl = threadIdx.x & (G - 1);
    const unsigned gm = __ballot_sync(0xffffffffu, greedy);
    mk = 0.f;
    s = 0.f;
    arg = 0;
    if (greedy) {
        Amax A{-INFINITY, 0x7fffffff, 0};
#pragma unroll
        for (int e = 0; e < E; ++e) amax_add(A, x[e], gl * E + e);
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(gm, A.best, o);
            const int oi = __shfl_xor_sync(gm, A.idx, o);
            const int on = __shfl_xor_sync(gm, A.nan, o);
            amax_merge(A, ob, oi, on);
        }
        arg = A.idx;
        bad = A.nan || A.best == INFINITY || A.best == -INFINITY;
    } else {
        const unsigned sm = ~gm;
        float m = x[0];
#pragma unroll
        for (int e = 1; e < E; ++e) m = fmaxf(m, x[e]);
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(sm, m, o));
        mk = (m > -INFINITY && m < INFINITY) ? ceilf(__fmul_rn(m, khi)) : 0.f;
        float t = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) t += scaled_exp(x[e], khi, klo, mk);
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1) t += __shfl_xor_sync(sm, t, o);
        s = t;
        bad = !(m > -INFINITY) || m == INFINITY || !isfinite(t) || !(t > 0.f);
    }
}

// Inclusive prefix over the G lanes of a group.
template <int G>
__device__ __forceinline__ double group_inclusive_scan(double x)
{
    const int gl = threadIdx.x & (G - 1);
#pragma unroll
    for (int o = 1; o < G; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, x, o, G);
        if (gl >= o) x += y;
    }
    return x;
}

template <int ESZ, int G, int E>
__device__ __forceinline__ void small_group(const TailArgs& a, int b, bool valid)
{
    const int gl = threadIdx.x & (G - 1);
    const int gamma = a.gamma, R = a.R;
    const float T = valid ? __ldg(a.temperature + b) : -1.f;
    const bool greedy = (T == 0.f);
    const bool tval = valid && temperature_ok(T);
    const int rows_used = !tval ? 0 : (greedy ? gamma + 1 : R);
    float khi = 0.f, klo = 0.f;
    if (tval && !greedy) split_k(T, &khi, &klo);

    // position j's inputs in lane j of the group
    const int x_j = (gl < gamma && tval) ? __ldg(a.tokens + (size_t)b * gamma + gl) : -1;
    const float u_j = (gl < gamma && valid) ? __ldg(a.u_accept + (size_t)b * gamma + gl) : 0.5f;
    const float ur = valid ? __ldg(a.u_resample + b) : 0.5f;

    // lane j: target row j and draft row j; every lane: the bonus row (gamma)
    float mk_t = 0.f, s_t = 0.f, mk_d = 0.f, s_d = 0.f, lt_j = 0.f, ld_j = 0.f, mk_b = 0.f, s_b = 0.f;
    int arg_t = 0, arg_b = 0, bad_any = 0;
    constexpr int RB = kSmallRegs / E > 0 ? kSmallRegs / E : 1;
    // fold rows [r0, r0 + RB) held in x
    auto fold_batch = [&](const float (&x)[RB][E], int r0) {
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = r0 + k;
            if (r >= R) break;
            float mk, s;
            int arg, bad;
            small_fold<G, E>(x[k], greedy, khi, klo, mk, s, arg, bad);
            if (r < rows_used) bad_any |= bad;
            const int j = r < gamma ? r : (r > gamma ? r - gamma - 1 : -1);
            float gv = 0.f;
            if (j >= 0) {
                // l[x_j] from the group lane that owns token x_j
                const int xj = __shfl_sync(0xffffffffu, x_j, j, G);
                const bool ok = xj >= 0 && xj < a.V;
                const int owner = ok ? xj / E : 0;
                gv = __shfl_sync(0xffffffffu, select_e<E>(x[k], ok ? xj - owner * E : 0), owner, G);
            }
            if (r == gamma) {
                mk_b = mk;
                s_b = s;
                arg_b = arg;
            } else if (gl == j) {
                if (r < gamma) {
                    mk_t = mk;
                    s_t = s;
                    arg_t = arg;
                    lt_j = gv;
                } else {
                    mk_d = mk;
                    s_d = s;
                    ld_j = gv;
                }
            }
        }
    };
    auto load_batch = [&](float (&x)[RB][E], int r0) {
#pragma unroll
        for (int k = 0; k < RB; ++k)
            if (r0 + k < R) small_load_row<ESZ, G, E>(a, b, r0 + k, r0 + k < rows_used, x[k]);
    };
    // two batches in flight: the next one loads while this one folds (R is the same
    // for every group, so every lane runs the same trip count)
    float xa[RB][E], xb[RB][E];
    load_batch(xa, 0);
    for (int r0 = 0; r0 < R; r0 += 2 * RB) {
        if (r0 + RB < R) load_batch(xb, r0 + RB);
        fold_batch(xa, r0);
        if (r0 + RB >= R) break;
        if (r0 + 2 * RB < R) load_batch(xa, r0 + 2 * RB);
        fold_batch(xb, r0 + RB);
    }

    // status, accept test, first rejection (per group)
    int st = 0;
    const unsigned badtok = group_bits<G>(__ballot_sync(0xffffffffu, gl < gamma && (x_j < 0 || x_j >= a.V)));
    const unsigned badu = group_bits<G>(__ballot_sync(
        0xffffffffu, !greedy && ((gl < gamma && !(u_j >= 0.f && u_j < 1.f)) || (gl == 0 && !(ur >= 0.f && ur < 1.f)))));
    if (!tval) {
        st = SV_ROW_BAD_TEMPERATURE;
    } else {
        if (badtok) st |= SV_ROW_BAD_TOKEN;
        if (bad_any) st |= SV_ROW_BAD_LOGITS;
        if (badu) st |= SV_ROW_BAD_UNIFORM;
    }
    const double a2_t = (double)mk_t + log2((double)s_t);
    const double a2_d = (double)mk_d + log2((double)s_d);
    bool acc = false;
    if (st == 0 && gl < gamma) {
        if (greedy) {
            acc = (x_j == arg_t);
        } else {
            const double rT = 1.0 / (double)T;
            const double lp = (double)lt_j * rT - a2_t * kLn2;
            const double lq = (double)ld_j * rT - a2_d * kLn2;
            acc = log((double)u_j) < (lp - lq);
        }
    }
    const unsigned mask = (gamma == 32) ? 0xffffffffu : ((1u << gamma) - 1u);
    const unsigned rej = group_bits<G>(__ballot_sync(0xffffffffu, !acc)) & mask;
    const int n = (st != 0) ? 0 : (rej ? __ffs(rej) - 1 : gamma);

    // the extra token: every lane takes part, groups that need no draw with dummies
    const bool bonus = (n == gamma);
    const bool draw = (st == 0) && !greedy;
    const int nl = n & (G - 1);
    const int arg_n = __shfl_sync(0xffffffffu, arg_t, nl, G);
    const float mkt_n = __shfl_sync(0xffffffffu, mk_t, nl, G);
    const float st_n = __shfl_sync(0xffffffffu, s_t, nl, G);
    const float mkd_n = __shfl_sync(0xffffffffu, mk_d, nl, G);
    const float sd_n = __shfl_sync(0xffffffffu, s_d, nl, G);
    SeqRec rec;
    rec.mode = bonus ? kModeBonus : kModeResidual;
    rec.n = n;
    rec.k_hi = khi;
    rec.k_lo = klo;
    rec.mk_t = bonus ? mk_b : mkt_n;
    rec.inv_s_t = draw ? (float)(1.0 / (double)(bonus ? s_b : st_n)) : 0.f;
    rec.mk_d = bonus ? 0.f : mkd_n;
    rec.inv_s_d = (draw && !bonus) ? (float)(1.0 / (double)sd_n) : 0.f;
    float xt[E], xd[E];
    small_load_row<ESZ, G, E>(a, b, n, draw, xt);
    small_load_row<ESZ, G, E>(a, b, gamma + 1 + n, draw && !bonus, xd);
    float w[E];
    double ls = 0.0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        w[e] = draw ? weight_of(rec, bonus, xt[e], bonus ? 0.f : xd[e]) : 0.f;
        ls += (double)w[e];
    }
    double incl = group_inclusive_scan<G>(ls);
    double S = __shfl_sync(0xffffffffu, incl, G - 1, G);
    // the residual vanished (below kResidualMin): draw from p_n instead
    const bool fb = draw && !bonus && !(S >= kResidualMin);
    if (__any_sync(0xffffffffu, fb)) {
        ls = 0.0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            w[e] = draw ? weight_of(rec, bonus || fb, xt[e], (bonus || fb) ? 0.f : xd[e]) : 0.f;
            ls += (double)w[e];
        }
        incl = group_inclusive_scan<G>(ls);
        S = __shfl_sync(0xffffffffu, incl, G - 1, G);
    }
    const double target = (double)ur * S;
    // the first lane whose running sum passes u*S, then the element inside it; if
    // rounding hides the crossing, the last token with a positive weight
    int hit = -1, lastpos = -1;
    double c = incl - ls;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        c += (double)w[e];
        if (hit < 0 && w[e] > 0.f && c > target) hit = gl * E + e;
        if (w[e] > 0.f) lastpos = gl * E + e;
    }
    const unsigned hm = group_bits<G>(__ballot_sync(0xffffffffu, hit >= 0));
    const unsigned lm = group_bits<G>(__ballot_sync(0xffffffffu, lastpos >= 0));
    const int hv = __shfl_sync(0xffffffffu, hit, hm ? __ffs(hm) - 1 : 0, G);
    const int lv = __shfl_sync(0xffffffffu, lastpos, lm ? 31 - __clz(lm) : 0, G);
    int extra = -1;
    if (st == 0) extra = greedy ? (bonus ? arg_b : arg_n) : (hm ? hv : (lm ? lv : -1));

    if (!valid) return;
    int32_t* ot = a.out_tokens + (size_t)b * (gamma + 1);
    for (int j = gl; j <= gamma; j += G) {
        int v = -1;
        if (st == 0) {
            if (j < n) v = x_j;  // j < n <= gamma <= G: lane j holds draft token j
            else if (j == n) v = extra;
        }
        ot[j] = v;
    }
    if (a.out_log_norm) {
        double* ln = a.out_log_norm + (size_t)b * R;
        const bool soft = tval && !greedy;
        if (gl < gamma) {
            ln[gl] = (soft && isfinite(a2_t) && s_t > 0.f) ? a2_t * kLn2 : (double)NAN;
            ln[gamma + 1 + gl] = (soft && isfinite(a2_d) && s_d > 0.f) ? a2_d * kLn2 : (double)NAN;
        }
        if (gl == 0) {
            const double a2_b = (double)mk_b + log2((double)s_b);
            ln[gamma] = (soft && isfinite(a2_b) && s_b > 0.f) ? a2_b * kLn2 : (double)NAN;
        }
    }
    if (gl == 0) {
        a.out_n[b] = n;
        if (a.out_status) a.out_status[b] = st | (fb ? SV_ROW_RESIDUAL_ZERO : 0);
    }
}

template <int ESZ, int G, int E>
__global__ void __launch_bounds__(kThreads, 4) sv_small(const __grid_constant__ TailArgs a, int B)
{
    constexpr int NG = 32 / G;  // sequences per warp
    const long long w = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const long long nw = (long long)gridDim.x * kWarps;
    const int grp = (threadIdx.x & 31) / G;
    for (long long base = w * NG; base < B; base += nw * NG) {
        const long long b = base + grp;
        small_group<ESZ, G, E>(a, (int)min(b, (long long)B - 1), b < B);
    }
}

}  // namespace sv
