// sv_topf.cuh -- the speculation cache's side of an outcome [Speculative
// Speculative Decoding, Metodologia 2, "Conceito Central" (the outcome is the
// number accepted plus one more token; the cache holds speculations for likely
// outcomes); Desafios 1 (a geometric fan-out over the accepted lengths) and 2
// (the extra token after a rejection comes from the residual, whose mass
// Saguaro sampling moves onto the cached top-F tokens)].
//
//   sv_topf          one CTA per (sequence b, outcome n with F_n > 0): the F_n
//                    most probable tokens of the distribution the extra token is
//                    drawn from after outcome n -- norm(max(0, p_n - q_n)) for
//                    n < gamma (p_n when the residual mass is below 2^-18, as the
//                    draw does), p_gamma for n = gamma, a point mass on the first
//                    argmax of target row n when T = 0 -- with their
//                    probabilities.  p and q come from the row log-normalisers
//                    spec_verify returned, so this is one more pass over the draw
//                    rows.  Each warp keeps the best F_n (weight, token) pairs of
//                    its part of the rows in its lanes (lane i: the i-th best,
//                    by weight, then smaller token); a candidate that beats lane
//                    F_n - 1 is inserted by one ballot and one shuffle.  The CTA
//                    then sorts the warps' 8 x 32 candidates (bitonic, shared
//                    memory) and keeps the first F_n.
//   sv_cache_lookup  one thread per sequence: the slot of outcome n's list that
//                    holds the extra token spec_verify emitted, else -1.
#pragma once

#include "sv_common.cuh"

namespace sv {

constexpr int kTopfThreads = 256;  // 3 CTAs per SM: 64 x 6 outcomes in one wave on 148 SMs
constexpr int kTopfWarps = kTopfThreads / 32;
constexpr int kTopfBatch = 4;  // 16-byte vectors per lane and row loaded before any is used

struct TopfArgs {
    const void* tgt;
    const void* dft;
    const float* temperature;
    const double* log_norm;     // [B][2*gamma+1] from spec_verify
    const int32_t* row_status;  // [B] from spec_verify
    int32_t* out_tokens;        // [B][Ftot]
    float* out_prob;            // [B][Ftot]
    int F[SV_MAX_GAMMA + 1];    // slots per outcome
    int off[SV_MAX_GAMMA + 2];  // first slot of each outcome
    int Ftot, B, gamma, V;
    int nz[SV_MAX_GAMMA + 1];   // the outcomes with F_n > 0, in order
    int n_nz;
};

// (aw, av) ranks before (bw, bv): larger weight, then smaller token
__device__ __forceinline__ bool ranks_before(float aw, int av, float bw, int bv)
{
    return aw > bw || (aw == bw && av < bv);
}

// Insert candidate (cw, cv), which ranks before lane F-1's pair, into the warp's
// list (lane i holds the i-th best); the last pair drops out.
__device__ __forceinline__ void list_insert(float& lw, int& lv, float cw, int cv, int F)
{
    const int lane = threadIdx.x & 31;
    const unsigned before = __ballot_sync(0xffffffffu, lane < F && ranks_before(lw, lv, cw, cv));
    const int pos = __popc(before);
    const float uw = __shfl_up_sync(0xffffffffu, lw, 1);
    const int uv = __shfl_up_sync(0xffffffffu, lv, 1);
    if (lane == pos) {
        lw = cw;
        lv = cv;
    } else if (lane > pos) {
        lw = uw;
        lv = uv;
    }
}

// The lane's candidates in w[0..VEC) (tokens i0 + e) that rank before the list's
// last pair, as a bit mask.
template <int VEC>
__device__ __forceinline__ unsigned qualifying(const float (&w)[VEC], int i0, float tw, int tv, float bar)
{
    unsigned qm = 0;
#pragma unroll
    for (int e = 0; e < VEC; ++e)
        if (w[e] > 0.f && w[e] >= bar && ranks_before(w[e], i0 + e, tw, tv)) qm |= 1u << e;
    return qm;
}

// Offer every qualifying candidate of the warp, one per round: the lowest lane
// that has one offers its first; the candidate is inserted if it still ranks
// before the list's last pair (the list may have moved on since the lane's vote),
// else dropped.  The final list does not depend on the order of the offers: the
// ranking is a total order.
template <int VEC>
__device__ __forceinline__ void list_offer_vec(float& lw, int& lv, float& tw, int& tv, const float (&w)[VEC],
                                               int i0, int F, unsigned qm, int* s_bar)
{
    const int lane = threadIdx.x & 31;
    unsigned m = __ballot_sync(0xffffffffu, qm != 0);
    if (!m) return;
    while (m) {
        const int src = __ffs(m) - 1;
        const int e0 = qm ? __ffs(qm) - 1 : 0;
        float cw = w[0];
#pragma unroll
        for (int e = 1; e < VEC; ++e)
            if (e == e0) cw = w[e];
        cw = __shfl_sync(0xffffffffu, cw, src);
        const int cv = __shfl_sync(0xffffffffu, i0 + e0, src);
        if (lane == src) qm &= ~(1u << e0);
        if (ranks_before(cw, cv, tw, tv)) {  // the same in every lane
            list_insert(lw, lv, cw, cv, F);
            tw = __shfl_sync(0xffffffffu, lw, F - 1);
            tv = __shfl_sync(0xffffffffu, lv, F - 1);
        }
        m = __ballot_sync(0xffffffffu, qm != 0);
    }
    // a full list's last weight bounds the CTA's F-th weight from below: publish it
    // (weights are >= 0, so their bit patterns order as integers)
    if (lane == 0 && tw > 0.f) atomicMax(s_bar, __float_as_int(tw));
}

// The F-th largest of the warp's 32 values (one per lane), by a bitonic sort in
// descending order across the lanes.  F <= 32.
__device__ __forceinline__ float warp_fth_largest(float v, int F)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const float o = __shfl_xor_sync(0xffffffffu, v, j);
            const bool keep_max = ((lane & j) == 0) == ((lane & k) == 0);
            v = keep_max ? fmaxf(v, o) : fminf(v, o);
        }
    return __shfl_sync(0xffffffffu, v, F - 1);
}

// The weights of row pair (t, d) at element i: max(0, p - q), or p (p_only),
// p = 2^(l*k_hi + l*k_lo - mt) * ct with mt an integer and ct = 2^(mt - a2_t).
struct TopfScale {
    float khi, klo, mt, ct, md, cd;
};

__device__ __forceinline__ float topf_weight(const TopfScale& z, bool p_only, float lt, float ld)
{
    const float p = ex2(__fmaf_rn(lt, z.klo, __fmaf_rn(lt, z.khi, -z.mt))) * z.ct;
    if (p_only) return p;
    const float q = ex2(__fmaf_rn(ld, z.klo, __fmaf_rn(ld, z.khi, -z.md))) * z.cd;
    return fmaxf(0.f, p - q);
}

// topf_weight for elements (0, 1) of a pair on packed fp32 pairs (every
// operation rounds as in topf_weight, so both give the same bits).
__device__ __forceinline__ void topf_weight2(const TopfScale& z, bool p_only, float lt0, float lt1, float ld0, float ld1,
                                             float& w0, float& w1)
{
    const unsigned long long KH = pack2(z.khi, z.khi), KL = pack2(z.klo, z.klo);
    const unsigned long long xt = pack2(lt0, lt1);
    float a0, a1;
    unpack2(fma2(xt, KL, fma2(xt, KH, pack2(-z.mt, -z.mt))), a0, a1);
    const unsigned long long P = mul2(pack2(ex2(a0), ex2(a1)), pack2(z.ct, z.ct));
    if (p_only) {
        unpack2(P, w0, w1);
        return;
    }
    const unsigned long long xd = pack2(ld0, ld1);
    float b0, b1;
    unpack2(fma2(xd, KL, fma2(xd, KH, pack2(-z.md, -z.md))), b0, b1);
    float d0, d1;
    unpack2(sub2(P, mul2(pack2(ex2(b0), ex2(b1)), pack2(z.cd, z.cd))), d0, d1);
    w0 = fmaxf(0.f, d0);
    w1 = fmaxf(0.f, d1);
}

// The sum of a vector's weights, as a short tree (4 or 8 elements).
template <int N>
__device__ __forceinline__ float tree8_any(const float (&w)[N])
{
    if (N == 8) return ((w[0] + w[1]) + (w[2] + w[3])) + ((w[4] + w[5]) + (w[6] + w[7]));
    return (w[0] + w[1]) + (w[2] + w[3]);
}

// One pass over the CTA's rows: every warp's list of its part, the fp64 total of
// the weights (block order), then the sorted CTA list in s_w / s_v.
template <int ESZ>
__device__ void topf_pass(const TopfArgs& g, const unsigned char* rt, const unsigned char* rd, bool p_only,
                          const TopfScale& z, int F, float* s_w, int* s_v, double* s_sum, int* s_bar, double& S)
{
    constexpr int VEC = 16 / ESZ;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int V = g.V;
    const bool vec = ((size_t)V * ESZ) % 16 == 0;
    float lw = -1.f, tw = -1.f;
    int lv = 0x7fffffff, tv = 0x7fffffff;
    double ls = 0.0;
    // a floor under this warp's candidates, from its first vectors: the F-th
    // largest of the 32 lanes' largest weights.  At least F weights reach it, so no
    // weight below it is among the CTA's F largest; it spares the rounds that an
    // empty list would otherwise spend on every positive weight.
    float floor_w = 0.f;
    bool seeded = false;
    if (vec) {
        const int nv = V / VEC;
        const int per = (nv + kTopfWarps - 1) / kTopfWarps;
        const int w0 = min(nv, warp * per), w1 = min(nv, w0 + per);
        // kTopfBatch vectors per lane and row in flight at once
        for (int q0 = w0; q0 < w1; q0 += 32 * kTopfBatch) {
            uint4 vt[kTopfBatch], vd[kTopfBatch];
#pragma unroll
            for (int u = 0; u < kTopfBatch; ++u) {
                const int q = q0 + u * 32 + lane;
                vt[u] = q < w1 ? __ldg(reinterpret_cast<const uint4*>(rt) + q) : make_uint4(0u, 0u, 0u, 0u);
                vd[u] = (q < w1 && !p_only) ? __ldg(reinterpret_cast<const uint4*>(rd) + q) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kTopfBatch; ++u) {
            const int q = q0 + u * 32 + lane;
            const bool ok = q < w1;
            float xt[VEC], xd[VEC];
            unpack<ESZ>(vt[u], xt);
            unpack<ESZ>(vd[u], xd);
            float w[VEC];
#pragma unroll
            for (int e = 0; e < VEC; e += 2) topf_weight2(z, p_only, xt[e], xt[e + 1], xd[e], xd[e + 1], w[e], w[e + 1]);
            if (!ok) {
#pragma unroll
                for (int e = 0; e < VEC; ++e) w[e] = 0.f;
            }
            ls += (double)tree8_any<VEC>(w);
            // one vote per vector; rounds only for the candidates that beat the list
            // and are not below another warp's published F-th weight (F pairs of that
            // warp outrank them).  The elements are tested only when the vector's
            // largest weight could qualify.
            float vmax = w[0];
#pragma unroll
            for (int e = 1; e < VEC; ++e) vmax = fmaxf(vmax, w[e]);
            if (!seeded) {  // the first vectors (uniform across the warp)
                floor_w = warp_fth_largest(vmax, F);
                seeded = true;
            }
            const float bar = fmaxf(__int_as_float(*reinterpret_cast<volatile int*>(s_bar)), floor_w);
            const unsigned qm = (vmax > 0.f && vmax >= bar && vmax >= tw) ? qualifying<VEC>(w, q * VEC, tw, tv, bar) : 0u;
            list_offer_vec<VEC>(lw, lv, tw, tv, w, q * VEC, F, qm, s_bar);
            }
        }
    } else {
        const int per = (V + kTopfWarps - 1) / kTopfWarps;
        const int e0 = min(V, warp * per), e1 = min(V, e0 + per);
        for (int i0 = e0; i0 < e1; i0 += 32) {
            const int i = i0 + lane;
            const bool ok = i < e1;
            const float lt = ok ? load_logit<ESZ>(rt, (size_t)i) : 0.f;
            const float ld = (ok && !p_only) ? load_logit<ESZ>(rd, (size_t)i) : 0.f;
            const float w1[1] = {ok ? topf_weight(z, p_only, lt, ld) : 0.f};
            ls += (double)w1[0];
            const float bar = __int_as_float(*reinterpret_cast<volatile int*>(s_bar));
            list_offer_vec<1>(lw, lv, tw, tv, w1, i, F, qualifying<1>(w1, i, tw, tv, bar), s_bar);
        }
    }
    // the total, in a fixed order: lanes, then warps
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
    if (lane == 0) s_sum[warp] = ls;
    s_w[tid] = lane < F ? lw : -1.f;
    s_v[tid] = lane < F ? lv : 0x7fffffff;
    __syncthreads();
    S = 0.0;
    for (int k = 0; k < kTopfWarps; ++k) S += s_sum[k];
    // bitonic sort of the kTopfThreads candidates, best first
    for (int k = 2; k <= kTopfThreads; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            const int ixj = tid ^ j;
            if (ixj > tid) {
                const float aw = s_w[tid], bw = s_w[ixj];
                const int av = s_v[tid], bv = s_v[ixj];
                const bool up = (tid & k) == 0;  // this block ends best first
                const bool swap = up ? ranks_before(bw, bv, aw, av) : ranks_before(aw, av, bw, bv);
                if (swap) {
                    s_w[tid] = bw;
                    s_v[tid] = bv;
                    s_w[ixj] = aw;
                    s_v[ixj] = av;
                }
            }
            __syncthreads();
        }
    }
}

template <int ESZ>
__global__ void __launch_bounds__(kTopfThreads, 3) sv_topf(const __grid_constant__ TopfArgs g)
{
    __shared__ float s_w[kTopfThreads];
    __shared__ int s_v[kTopfThreads];
    __shared__ double s_sum[kTopfWarps];
    __shared__ int s_arg;
    __shared__ int s_bar[1];  // bits of the largest F-th weight any warp has published
    const int tid = threadIdx.x, lane = tid & 31;
    const int b = blockIdx.x / g.n_nz;
    const int n = g.nz[blockIdx.x - b * g.n_nz];
    const int gamma = g.gamma, R = 2 * gamma + 1, F = g.F[n];
    int32_t* ot = g.out_tokens + (size_t)b * g.Ftot + g.off[n];
    float* op = g.out_prob + (size_t)b * g.Ftot + g.off[n];
    const float T = __ldg(g.temperature + b);
    const int st = __ldg(g.row_status + b);
    // a sequence with an invalid temperature or a bad row has no distributions
    bool bad = (st & (SV_ROW_BAD_TEMPERATURE | SV_ROW_BAD_LOGITS)) != 0 || !temperature_ok(T);
    const double* ln = g.log_norm + (size_t)b * R;
    if (!bad && T != 0.f)
        for (int r = 0; r < R; ++r) bad = bad || !isfinite(__ldg(ln + r));
    if (bad) {
        for (int s = tid; s < F; s += kTopfThreads) {
            ot[s] = -1;
            op[s] = 0.f;
        }
        return;
    }
    const size_t rowb = (size_t)g.V * ESZ;
    const unsigned char* rt = static_cast<const unsigned char*>(g.tgt) + ((size_t)b * (gamma + 1) + n) * rowb;
    if (T == 0.f) {
        // a point mass on the first argmax of target row n
        Amax A{-INFINITY, 0x7fffffff, 0};
        for (int i = tid; i < g.V; i += kTopfThreads) amax_add(A, load_logit<ESZ>(rt, (size_t)i), i);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, A.best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, A.idx, o);
            const int on = __shfl_xor_sync(0xffffffffu, A.nan, o);
            amax_merge(A, ob, oi, on);
        }
        // the warps' maxima, merged in warp order (each warp saw interleaved indices,
        // so the merge keeps the best value's smallest index)
        if (lane == 0) {
            s_w[tid >> 5] = A.best;
            s_v[tid >> 5] = A.idx;
        }
        __syncthreads();
        if (tid == 0) {
            Amax B{-INFINITY, 0x7fffffff, 0};
            for (int k = 0; k < kTopfWarps; ++k) amax_merge(B, s_w[k], s_v[k], 0);
            s_arg = B.idx;
        }
        __syncthreads();
        for (int s = tid; s < F; s += kTopfThreads) {
            ot[s] = s == 0 ? s_arg : -1;
            op[s] = s == 0 ? 1.f : 0.f;
        }
        return;
    }
    const unsigned char* rd = n < gamma ? static_cast<const unsigned char*>(g.dft) + ((size_t)b * gamma + n) * rowb
                                        : rt;
    TopfScale z;
    split_k(T, &z.khi, &z.klo);
    {
        // p_v = 2^(l_v*k - a2) with a2 = lse*log2(e): the integer part of a2 is the
        // offset, the rest a factor in [1, 2)
        const double a2t = __ldg(ln + n) * kLog2e;
        const double ft = floor(a2t);
        z.mt = (float)ft;
        z.ct = (float)exp2(ft - a2t);
        z.md = 0.f;
        z.cd = 0.f;
        if (n < gamma) {
            const double a2d = __ldg(ln + gamma + 1 + n) * kLog2e;
            const double fd = floor(a2d);
            z.md = (float)fd;
            z.cd = (float)exp2(fd - a2d);
        }
    }
    double S;
    bool p_only = (n == gamma);
    if (tid == 0) *s_bar = 0;
    __syncthreads();
    topf_pass<ESZ>(g, rt, rd, p_only, z, F, s_w, s_v, s_sum, s_bar, S);
    if (!p_only && !(S >= kResidualMin)) {
        // the residual vanished (below kResidualMin): p_n, as the draw
        __syncthreads();
        if (tid == 0) *s_bar = 0;
        __syncthreads();
        topf_pass<ESZ>(g, rt, rd, true, z, F, s_w, s_v, s_sum, s_bar, S);
    }
    for (int s = tid; s < F; s += kTopfThreads) {
        const float w = s_w[s];
        ot[s] = w > 0.f ? s_v[s] : -1;
        op[s] = w > 0.f ? (float)((double)w / S) : 0.f;
    }
}

// The slot of each sequence's outcome (n, extra token) in its cache, else -1.
__global__ void sv_cache_lookup(const int32_t* __restrict__ out_tokens, const int32_t* __restrict__ out_n,
                                const int32_t* __restrict__ cache, const __grid_constant__ TopfArgs g,
                                int32_t* __restrict__ out_slot)
{
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= g.B) return;
    int slot = -1;
    const int n = __ldg(out_n + b);
    if (n >= 0 && n <= g.gamma) {
        const int x = __ldg(out_tokens + (size_t)b * (g.gamma + 1) + n);
        if (x >= 0)
            for (int s = g.off[n]; s < g.off[n + 1] && slot < 0; ++s)
                if (__ldg(cache + (size_t)b * g.Ftot + s) == x) slot = s;
    }
    out_slot[b] = slot;
}

}  // namespace sv
