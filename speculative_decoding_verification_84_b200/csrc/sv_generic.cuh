// sv_generic.cuh -- the any-shape path: two kernels, one CTA per work chunk.
//
//   sv_rowpass   one CTA per (sequence, row, vocabulary chunk): streams the
//                chunk once with 128-bit loads (unaligned rows get a scalar
//                head and tail), reduces it to a Partial, and takes a ticket
//                on the sequence; the last CTA runs sequence_tail.
//   sv_resample  one CTA per (sequence, chunk) of the sequences that need a
//                sampled token: chunk sums of the residual (or bonus) weights;
//                the last CTA of a sequence finds u*S with block prefix scans
//                over chunk sums and then inside the chosen chunk.
//                [Speculative Speculative Decoding, Metodologia 2: outcome =
//                accepted count + extra token; residual distribution.]
// Used when rows are not 16-byte aligned or are too short for the streaming
// kernels in sv_pass.cuh.
#pragma once

#include "sv_common.cuh"

namespace sv {

constexpr int kUnroll = 4;

struct GenericArgs {
    TailArgs t;
    Partial* part;  // writable alias of t.part
    int nc1, C1;
    // pass 2
    const float* u_resample;
    unsigned* ticket2;
    double* rsum;
    int nc2, C2;
};

// Zero the call's tickets (n 16-byte words).  The general path
// counts arrivals per sequence; starting every call from zero means a workspace
// carries nothing from one call to the next.
__global__ void __launch_bounds__(256) sv_reset(uint4* p, long long n)
{
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        p[i] = make_uint4(0u, 0u, 0u, 0u);
}

template <int ESZ, bool GREEDY>
__device__ __forceinline__ void scan_chunk(const unsigned char* rowp, int v0, int v1, float khi,
                                           float klo, Lse& L, Amax& A)
{
    constexpr int VEC = 16 / ESZ;
    const unsigned char* cp = rowp + (size_t)v0 * ESZ;
    const int n = v1 - v0;
    int head = (int)(((16u - ((uintptr_t)cp & 15u)) & 15u) / ESZ);
    if (head > n) head = n;
    const int nvec = (n - head) / VEC;
    const int tail = n - head - nvec * VEC;
    const uint4* vp = reinterpret_cast<const uint4*>(cp + (size_t)head * ESZ);
    const int tid = threadIdx.x;
    const int vbase = v0 + head;

    int i = tid;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (; i + (kUnroll - 1) * kThreads < nvec; i += kUnroll * kThreads) {
        uint4 r[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) r[u] = ld_stream(vp + i + u * kThreads);
        if (GREEDY) {
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                float x[VEC];
                unpack<ESZ>(r[u], x);
                const int e0 = vbase + (i + u * kThreads) * VEC;
#pragma unroll
                for (int e = 0; e < VEC; ++e) amax_add(A, x[e], e0 + e);
            }
        } else {
            lse_group<ESZ, kUnroll>(L, acc, r, khi, klo);
        }
    }
    if (!GREEDY) lse_fold(L, acc);
    for (; i < nvec; i += kThreads) {
        float x[VEC];
        unpack<ESZ>(ld_stream(vp + i), x);
        if (GREEDY) {
            const int e0 = vbase + i * VEC;
#pragma unroll
            for (int e = 0; e < VEC; ++e) amax_add(A, x[e], e0 + e);
        } else {
            lse_add<VEC>(L, x, khi, klo);
        }
    }
    // unaligned head and ragged tail, one element per thread
    int e = -1;
    if (tid < head) e = v0 + tid;
    else if (tid >= 32 && tid - 32 < tail) e = vbase + nvec * VEC + (tid - 32);
    if (e >= 0) {
        const float x = load_logit<ESZ>(rowp, (size_t)e);
        if (GREEDY) amax_add(A, x, e);
        else lse_add<1>(L, &x, khi, klo);
    }
}

// Reduce per-thread softmax state over kThreads threads into one Partial (thread 0).
template <class SYNC>
__device__ Partial reduce_lse(Lse L, float* s_red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float om = __shfl_xor_sync(0xffffffffu, L.m, o);
        const float omk = __shfl_xor_sync(0xffffffffu, L.mk, o);
        const float os = __shfl_xor_sync(0xffffffffu, L.s, o);
        lse_merge(L, om, omk, os);
    }
    SYNC::sync();
    if (lane == 0) {
        s_red[warp] = L.m;
        s_red[kWarps + warp] = L.mk;
        s_red[2 * kWarps + warp] = L.s;
    }
    SYNC::sync();
    Partial out{0.f, 0.f, 0.f, 0};
    if (threadIdx.x == 0) {
        Lse F;
        lse_init(F);
        for (int w = 0; w < kWarps; ++w) lse_merge(F, s_red[w], s_red[kWarps + w], s_red[2 * kWarps + w]);
        out.m = F.m;
        out.mk = F.mk;
        out.s = F.s;
    }
    return out;
}

template <class SYNC>
__device__ Partial reduce_amax(Amax A, float* s_red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, A.best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, A.idx, o);
        const int on = __shfl_xor_sync(0xffffffffu, A.nan, o);
        amax_merge(A, ob, oi, on);
    }
    SYNC::sync();
    if (lane == 0) {
        s_red[warp] = A.best;
        s_red[kWarps + warp] = __int_as_float(A.idx);
        s_red[2 * kWarps + warp] = (float)A.nan;
    }
    SYNC::sync();
    Partial out{0.f, 0.f, 0.f, 0};
    if (threadIdx.x == 0) {
        Amax F{-INFINITY, 0x7fffffff, 0};
        for (int w = 0; w < kWarps; ++w)
            amax_merge(F, s_red[w], __float_as_int(s_red[kWarps + w]), s_red[2 * kWarps + w] != 0.f);
        out.m = F.best;
        out.s = (float)F.nan;
        out.idx = F.idx;
    }
    return out;
}

template <int ESZ>
__global__ void __launch_bounds__(kThreads) sv_rowpass(GenericArgs g)
{
    __shared__ float s_red[3 * kWarps];
    __shared__ int s_last;
    __shared__ TailSmem s_tail;
    const TailArgs& a = g.t;

    const int c = blockIdx.x % g.nc1;
    const int rr = blockIdx.x / g.nc1;
    const int r = rr % a.R;
    const int b = rr / a.R;
    const float T = a.temperature[b];
    const bool tval = temperature_ok(T);
    const bool greedy = (T == 0.f);
    const bool active = tval && !(greedy && r > a.gamma);

    if (active) {
        const size_t V = (size_t)a.V;
        const unsigned char* rowp =
            r <= a.gamma
                ? static_cast<const unsigned char*>(a.tgt) + ((size_t)b * (a.gamma + 1) + r) * V * ESZ
                : static_cast<const unsigned char*>(a.dft) + ((size_t)b * a.gamma + (r - a.gamma - 1)) * V * ESZ;
        const int v0 = c * g.C1;
        const int v1 = min(a.V, v0 + g.C1);
        Partial out;
        Lse L;
        lse_init(L);
        Amax A{-INFINITY, 0x7fffffff, 0};
        if (greedy) {
            scan_chunk<ESZ, true>(rowp, v0, v1, 0.f, 0.f, L, A);
            out = reduce_amax<BlockSync>(A, s_red);
        } else {
            float khi, klo;
            split_k(T, &khi, &klo);
            scan_chunk<ESZ, false>(rowp, v0, v1, khi, klo, L, A);
            out = reduce_lse<BlockSync>(L, s_red);
        }
        if (threadIdx.x == 0) g.part[((size_t)b * a.R + r) * g.nc1 + c] = out;
    }

    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&a.ticket[b], 1u);
        s_last = (prev == (unsigned)(a.R * g.nc1 - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    sequence_tail<ESZ, kThreads, BlockSync>(a, b, threadIdx.x, FloatPartials{a.part}, s_tail);
}

// Sum of the weights over [v0, v1) (valid in thread 0).
template <int ESZ>
__device__ double chunk_weight_sum(const unsigned char* trow, const unsigned char* drow, const SeqRec& s,
                                   bool p_only, int v0, int v1, double* sm)
{
    constexpr int VEC = 16 / ESZ;
    const int tid = threadIdx.x;
    const int n = v1 - v0;
    const unsigned char* tp = trow + (size_t)v0 * ESZ;
    const unsigned char* dp = p_only ? nullptr : drow + (size_t)v0 * ESZ;
    // chunk starts are multiples of 8 elements, so a chunk is 16-byte aligned
    // exactly when its row is; misaligned rows take the scalar path
    const bool vec_ok = (((uintptr_t)tp & 15u) == 0) && (p_only || (((uintptr_t)dp & 15u) == 0));
    double acc = 0.0;
    int done = 0;
    if (vec_ok) {
        const int nvec = n / VEC;
        const uint4* tv = reinterpret_cast<const uint4*>(tp);
        const uint4* dv = reinterpret_cast<const uint4*>(dp);
        for (int i = tid; i < nvec; i += kThreads) {
            float xt[VEC], xd[VEC];
            unpack<ESZ>(ld_stream(tv + i), xt);
            if (!p_only) unpack<ESZ>(ld_stream(dv + i), xd);
            float w[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int e = 0; e < VEC; ++e) w[e] = weight_of(s, p_only, xt[e], p_only ? 0.f : xd[e]);
            acc += (double)tree8(w);
        }
        done = nvec * VEC;
    }
    for (int e = done + tid; e < n; e += kThreads) {
        const float lt = load_logit<ESZ>(trow, (size_t)(v0 + e));
        const float ld = p_only ? 0.f : load_logit<ESZ>(drow, (size_t)(v0 + e));
        acc += (double)weight_of(s, p_only, lt, ld);
    }
    return block_sum<BlockSync>(acc, sm);
}

// Inverse CDF over the sequence's weights, given the per-chunk sums in rs[]:
// the smallest token k with running sum C_k > u * S; if rounding leaves none,
// the last token with a positive weight.
template <int ESZ>
__device__ void sequence_draw(const GenericArgs& g, int b, const SeqRec& s, const unsigned char* trow,
                              const unsigned char* drow)
{
    __shared__ double s_scan[kWarps];
    __shared__ double s_bcast;
    __shared__ int s_found, s_lastpos;

    const int tid = threadIdx.x;
    const int nc = g.nc2, C = g.C2, V = g.t.V;
    double* rs = g.rsum + (size_t)b * nc;
    bool p_only = (s.mode == kModeBonus);

    // total mass, in the same tile-scan order that the chunk search below uses
    double S = 0.0;
    for (int c0 = 0; c0 < nc; c0 += kThreads) {
        double tot;
        block_inclusive_scan<BlockSync>((c0 + tid < nc) ? __ldcg(rs + c0 + tid) : 0.0, s_scan, &tot);
        S += tot;
    }
    int flag = 0;
    if (!(S >= kResidualMin) && s.mode == kModeResidual) {
        // the residual vanished (below kResidualMin): draw from p_n instead
        flag = SV_ROW_RESIDUAL_ZERO;
        p_only = true;
        for (int c = 0; c < nc; ++c) {
            const double cs = chunk_weight_sum<ESZ>(trow, nullptr, s, true, c * C, min(V, (c + 1) * C), s_scan);
            if (tid == 0) rs[c] = cs;
        }
        __threadfence_block();
        __syncthreads();
        S = 0.0;
        for (int c0 = 0; c0 < nc; c0 += kThreads) {
            double tot;
            block_inclusive_scan<BlockSync>((c0 + tid < nc) ? rs[c0 + tid] : 0.0, s_scan, &tot);
            S += tot;
        }
    }
    const double target = (double)g.u_resample[b] * S;

    // 1) the chunk c* holding the target: first chunk whose inclusive prefix > target
    if (tid == 0) { s_found = 0x7fffffff; s_lastpos = -1; s_bcast = 0.0; }
    __syncthreads();
    double carry = 0.0;
    int cstar = -1;
    for (int c0 = 0; c0 < nc; c0 += kThreads) {
        const int c = c0 + tid;
        const double v = (c < nc) ? __ldcg(rs + c) : 0.0;
        double tot;
        const double incl = carry + block_inclusive_scan<BlockSync>(v, s_scan, &tot);
        const bool hit = (c < nc) && (incl > target);
        if (hit) atomicMin(&s_found, c);
        if (c < nc && v > 0.0) atomicMax(&s_lastpos, c);
        __syncthreads();
        if (hit && c == s_found) s_bcast = incl - v;  // exclusive prefix before c*
        __syncthreads();
        if (s_found != 0x7fffffff) { cstar = s_found; break; }
        carry += tot;
    }
    const bool take_last = (cstar < 0);
    const double base = take_last ? 0.0 : s_bcast;
    if (take_last) cstar = s_lastpos;
    __syncthreads();

    // 2) the token inside c*: thread t owns elements [t*E, t*E + E) of each tile
    constexpr int E = 8;
    const int v0 = cstar < 0 ? 0 : cstar * C;
    const int v1 = cstar < 0 ? 0 : min(V, v0 + C);
    if (tid == 0) { s_found = 0x7fffffff; s_lastpos = -1; }
    __syncthreads();
    double run = base;
    for (int t0 = v0; t0 < v1; t0 += kThreads * E) {
        const int e0 = t0 + tid * E;
        float w[E];
        double loc = 0.0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int v = e0 + e;
            float x = 0.f;
            if (v < v1) {
                const float lt = load_logit<ESZ>(trow, (size_t)v);
                const float ld = p_only ? 0.f : load_logit<ESZ>(drow, (size_t)v);
                x = weight_of(s, p_only, lt, ld);
            }
            w[e] = x;
            loc += (double)x;
        }
        double tot;
        double c = run + block_inclusive_scan<BlockSync>(loc, s_scan, &tot) - loc;
        int hit = -1, lastpos = -1;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            c += (double)w[e];
            if (hit < 0 && w[e] > 0.f && c > target) hit = e0 + e;
            if (w[e] > 0.f) lastpos = e0 + e;
        }
        if (!take_last && hit >= 0) atomicMin(&s_found, hit);
        if (lastpos >= 0) atomicMax(&s_lastpos, lastpos);
        __syncthreads();
        if (s_found != 0x7fffffff) break;
        run += tot;
    }
    __syncthreads();
    if (tid == 0) {
        const int k = (s_found != 0x7fffffff) ? s_found : s_lastpos;
        g.t.out_tokens[(size_t)b * (g.t.gamma + 1) + s.n] = k;
        if (flag && g.t.out_status) g.t.out_status[b] |= flag;
    }
}

template <int ESZ>
__global__ void __launch_bounds__(kThreads) sv_resample(GenericArgs g)
{
    __shared__ double s_red[kWarps];
    __shared__ int s_last;

    const int c = blockIdx.x % g.nc2;
    const int b = blockIdx.x / g.nc2;
    const SeqRec s = g.t.seq[b];
    if (s.mode == kModeNone) return;

    const size_t V = (size_t)g.t.V;
    const unsigned char* trow = static_cast<const unsigned char*>(g.t.tgt) +
                                ((size_t)b * (g.t.gamma + 1) + s.n) * V * ESZ;
    const unsigned char* drow = s.mode == kModeResidual
                                    ? static_cast<const unsigned char*>(g.t.dft) + ((size_t)b * g.t.gamma + s.n) * V * ESZ
                                    : nullptr;
    const int v0 = c * g.C2;
    const int v1 = min(g.t.V, v0 + g.C2);
    const double cs = chunk_weight_sum<ESZ>(trow, drow, s, s.mode == kModeBonus, v0, v1, s_red);
    if (threadIdx.x == 0) {
        g.rsum[(size_t)b * g.nc2 + c] = cs;
        __threadfence();
        const unsigned prev = atomicAdd(&g.ticket2[b], 1u);
        s_last = (prev == (unsigned)(g.nc2 - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    sequence_draw<ESZ>(g, b, s, trow, drow);
}

}  // namespace sv
