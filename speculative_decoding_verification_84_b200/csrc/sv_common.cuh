// sv_common.cuh -- device helpers shared by the spec_verify kernels (sm_100a).
//
// Arithmetic conventions (both kernel families use exactly these helpers):
//   * k = log2(e) / T is split as k_hi + k_lo with k_hi = k rounded toward zero
//     and k_lo > 0, so l*k is formed as fma(l, k_lo, fma(l, k_hi, -off)) without
//     a rounded 1/T biasing the normaliser, and -inf logits give -inf exponents
//     (never -inf + inf).
//   * Row normalisers are kept as (m, mk, s): m the largest logit seen, mk =
//     ceil(m * k_hi) an integer offset, s = sum of 2^(l*k - mk).  Every rescale
//     multiplies by 2^(integer), which is exact.
//   * Temperature before the log-softmax, log-space test [FlashSpec, Metodologia
//     1, "Estabilidade Numerica"].
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <float.h>
#include <math.h>
#include <stdint.h>

#include "spec_verify.h"

namespace sv {

constexpr int kThreads = 256;            // threads that compute (generic CTA / stream consumers)
constexpr int kWarps = kThreads / 32;
constexpr int kMaxRows = 2 * SV_MAX_GAMMA + 1;
constexpr double kLn2 = 0.69314718055994530942;
// A residual mass below this counts as vanished and the extra token is drawn
// from p_n instead (row-status bit 8): at this size the residual is below what
// fp32 weights resolve, and the cases that reach it (q_n equal to p_n up to a
// shift of the normaliser) have a residual proportional to p_n.
constexpr double kResidualMin = 0x1p-18;
constexpr double kLog2e = 1.44269504088896340736;

enum : int { kModeNone = 0, kModeResidual = 1, kModeBonus = 2 };

// Partial result of one (row, chunk).  Softmax rows: m = max logit, mk = integer
// offset ceil(m * k_hi), s = sum of 2^(l*k - mk).  Greedy rows: m = max,
// idx = first index of the max, s != 0 if a NaN was seen.
struct __align__(16) Partial {
    float m;
    float mk;
    float s;
    int idx;
};

// What the draw needs about one sequence.
struct __align__(16) SeqRec {
    int mode;
    int n;
    float mk_t;     // integer offset of target row n
    float inv_s_t;  // 1 / sum of target row n
    float mk_d;     // same for draft row n
    float inv_s_d;
    float k_hi;     // log2(e)/T = k_hi + k_lo
    float k_lo;
};

// Barrier policy of sequence_tail's callers: the whole CTA.
struct BlockSync {
    static __device__ __forceinline__ void sync() { __syncthreads(); }
};

// ----------------------------------------------------------------------------- loads and math

__device__ __forceinline__ uint4 ld_stream(const uint4* p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float ex2(float x)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// 2^d for an integer-valued d <= 0, exactly (0 below the normal range)
__device__ __forceinline__ float pow2i(float d)
{
    return d >= -126.f ? __int_as_float(((int)d + 127) << 23) : 0.f;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <int ESZ>
__device__ __forceinline__ float load_logit(const void* base, size_t i)
{
    if (ESZ == 4) return __ldg((const float*)base + i);
    unsigned short h = __ldg((const unsigned short*)base + i);
    return __uint_as_float((uint32_t)h << 16);
}

template <int ESZ>
__device__ __forceinline__ void unpack(const uint4& v, float* x)
{
    if (ESZ == 2) {
        x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x); x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
        x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z); x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
    } else {
        x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
        x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
    }
}

// largest value of a 16-byte vector (NaN ignored unless all are NaN)
template <int ESZ>
__device__ __forceinline__ float vec_max(const uint4& v)
{
    if (ESZ == 2) {
        const __nv_bfloat162 a = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&v.x),
                                         *reinterpret_cast<const __nv_bfloat162*>(&v.y));
        const __nv_bfloat162 b = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&v.z),
                                         *reinterpret_cast<const __nv_bfloat162*>(&v.w));
        const __nv_bfloat162 c = __hmax2(a, b);
        const uint32_t w = *reinterpret_cast<const uint32_t*>(&c);
        return fmaxf(bf16_lo(w), bf16_hi(w));
    } else {
        return fmaxf(fmaxf(__uint_as_float(v.x), __uint_as_float(v.y)),
                     fmaxf(__uint_as_float(v.z), __uint_as_float(v.w)));
    }
}

// ---- online log-sum-exp state with integer offsets
struct Lse {
    float m, mk, s;
};

__device__ __forceinline__ void lse_init(Lse& a) { a.m = -INFINITY; a.mk = 0.f; a.s = 0.f; }

__device__ __forceinline__ void lse_rebase(Lse& a, float vmax, float khi)
{
    if (vmax > a.m) {
        const float mk = ceilf(__fmul_rn(vmax, khi));
        a.s = (a.m == -INFINITY) ? 0.f : a.s * pow2i(a.mk - mk);
        a.m = vmax;
        a.mk = mk;
    }
}

// 2^(x*k - off) with k = khi + klo (klo > 0): -inf maps to 0, NaN stays NaN
__device__ __forceinline__ float scaled_exp(float x, float khi, float klo, float off)
{
    return ex2(__fmaf_rn(x, klo, __fmaf_rn(x, khi, -off)));
}

template <int N>
__device__ __forceinline__ void lse_add(Lse& a, const float* x, float khi, float klo)
{
    float vm = x[0];
#pragma unroll
    for (int i = 1; i < N; ++i) vm = fmaxf(vm, x[i]);
    lse_rebase(a, vm, khi);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < N; ++i) acc += scaled_exp(x[i], khi, klo, a.mk);
    a.s += acc;
}

// Several 16-byte vectors at once: one max and at most one rescale for the group,
// then every term into one of 8 independent accumulators (short dependency
// chains).  acc[] holds sums relative to a.mk; fold them with lse_fold().
template <int ESZ, int NV>
__device__ __forceinline__ void lse_group(Lse& a, float* acc, const uint4* v, float khi, float klo)
{
    constexpr int VEC = 16 / ESZ;
    float vm = vec_max<ESZ>(v[0]);
#pragma unroll
    for (int u = 1; u < NV; ++u) vm = fmaxf(vm, vec_max<ESZ>(v[u]));
    if (vm > a.m) {
        const float mk = ceilf(__fmul_rn(vm, khi));
        const float f = (a.m == -INFINITY) ? 0.f : pow2i(a.mk - mk);  // mk never decreases
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= f;
        a.m = vm;
        a.mk = mk;
    }
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        float x[VEC];
        unpack<ESZ>(v[u], x);
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[(u * VEC + e) & 7] += scaled_exp(x[e], khi, klo, a.mk);
    }
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic: two IEEE fp32 operations per
// instruction, each rounded exactly like its scalar form)
__device__ __forceinline__ unsigned long long pack2(float a, float b)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ void unpack2(unsigned long long v, float& a, float& b)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}

__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ unsigned long long sub2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// lse_group with the exponent arguments and the accumulations done on packed
// pairs.  Element e of a vector still goes to acc[e & 7] in the same order, and
// every operation rounds as in lse_group, so the two give identical bits; this
// one issues about 3.5 instructions per element instead of 5.
template <int ESZ, int NV>
__device__ __forceinline__ void lse_group2(Lse& a, float* acc, const uint4* v, float khi, float klo)
{
    float vm = vec_max<ESZ>(v[0]);
#pragma unroll
    for (int u = 1; u < NV; ++u) vm = fmaxf(vm, vec_max<ESZ>(v[u]));
    if (vm > a.m) {
        const float mk = ceilf(__fmul_rn(vm, khi));
        const float f = (a.m == -INFINITY) ? 0.f : pow2i(a.mk - mk);  // mk never decreases
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= f;
        a.m = vm;
        a.mk = mk;
    }
    const unsigned long long KH = pack2(khi, khi), KL = pack2(klo, klo), NM = pack2(-a.mk, -a.mk);
    unsigned long long acc2[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) acc2[w] = pack2(acc[2 * w], acc[2 * w + 1]);
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const unsigned wd[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            // bf16: the word holds elements 2w (low half) and 2w+1; fp32: one element
            // per word, so words w and w+... pair as elements (u*4 + w) -> acc[(u*4+w) & 7]
            if (ESZ == 2) {
                const unsigned long long x2 = pack2(bf16_lo(wd[w]), bf16_hi(wd[w]));
                const unsigned long long y2 = fma2(x2, KL, fma2(x2, KH, NM));
                float y0, y1;
                unpack2(y2, y0, y1);
                acc2[w] = add2(acc2[w], pack2(ex2(y0), ex2(y1)));
            }
        }
        if (ESZ == 4) {
            // elements u*4 .. u*4+3 go to acc[(u*4 + i) & 7]: pairs (0,1), (2,3) of the
            // vector land in accumulator pairs ((u&1)*2 + 0) and ((u&1)*2 + 1)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const unsigned long long x2 = pack2(__uint_as_float(wd[2 * h]), __uint_as_float(wd[2 * h + 1]));
                const unsigned long long y2 = fma2(x2, KL, fma2(x2, KH, NM));
                float y0, y1;
                unpack2(y2, y0, y1);
                const int w = (u & 1) * 2 + h;
                acc2[w] = add2(acc2[w], pack2(ex2(y0), ex2(y1)));
            }
        }
    }
#pragma unroll
    for (int w = 0; w < 4; ++w) unpack2(acc2[w], acc[2 * w], acc[2 * w + 1]);
}

__device__ __forceinline__ void lse_fold(Lse& a, const float* acc)
{
    a.s += ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

// ---- online log-sum-exp with a lagging offset
//
// The streaming pass keeps, per warp, one offset mk (an integer, carried from
// segment to segment) and per-lane accumulators of 2^(l*k - mk) on packed fp32
// pairs.  Unlike lse_group2 it takes no maximum in the loop: every term is formed
// against the offset already held.  The segment's sum is checked once at its
// end: outside [2^-40, 2^100) (a term far above the offset or an overflow, a
// carried offset far above this row's values, NaN, an all -inf segment) the
// segment is summed again exactly (maximum first) -- rare, and the data is then
// mostly in L2.  Inside that range no term overflowed and terms down to 2^-126
// against the offset (at most 2^-86 of the sum) were kept, so the relative
// precision is that of the exact form.

// Exponentials of NV vectors against offset mk, added into 4 packed pairs acc.
// bf16: word w of a vector holds elements 2w, 2w+1 -> pair w.  fp32: elements
// (0,1) and (2,3) of vector u -> pairs 2(u&1), 2(u&1)+1.
template <int ESZ, int NV>
__device__ __forceinline__ void lazy_exps_add(unsigned long long* acc, const uint4* v, float khi, float klo, float mk)
{
    const unsigned long long KH = pack2(khi, khi), KL = pack2(klo, klo), NM = pack2(-mk, -mk);
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const unsigned wd[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        if (ESZ == 2) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const unsigned long long x2 = pack2(bf16_lo(wd[w]), bf16_hi(wd[w]));
                const unsigned long long y2 = fma2(x2, KL, fma2(x2, KH, NM));
                float y0, y1;
                unpack2(y2, y0, y1);
                acc[w] = add2(acc[w], pack2(ex2(y0), ex2(y1)));
            }
        } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const unsigned long long x2 = pack2(__uint_as_float(wd[2 * h]), __uint_as_float(wd[2 * h + 1]));
                const unsigned long long y2 = fma2(x2, KL, fma2(x2, KH, NM));
                float y0, y1;
                unpack2(y2, y0, y1);
                const int w = (u & 1) * 2 + h;
                acc[w] = add2(acc[w], pack2(ex2(y0), ex2(y1)));
            }
        }
    }
}

// Sum of a warp's accumulators (all lanes against the same offset), in every lane.
__device__ __forceinline__ float lazy_warp_sum(const unsigned long long* acc)
{
    float a[8];
#pragma unroll
    for (int w = 0; w < 4; ++w) unpack2(acc[w], a[2 * w], a[2 * w + 1]);
    float s = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// 2^d in double for an integer-valued d <= 0 (exact; 0 below the normal range)
__device__ __forceinline__ double pow2d(float d)
{
    return d >= -1022.f ? __longlong_as_double((long long)((int)d + 1023) << 52) : 0.0;
}

// Sum of 8 residual / bonus weights, as a short tree.
__device__ __forceinline__ float tree8(const float* w)
{
    return ((w[0] + w[1]) + (w[2] + w[3])) + ((w[4] + w[5]) + (w[6] + w[7]));
}

__device__ __forceinline__ void lse_merge(Lse& a, float m, float mk, float s)
{
    if (m == -INFINITY) return;
    if (a.m == -INFINITY) { a.m = m; a.mk = mk; a.s = s; return; }
    const float MK = fmaxf(a.mk, mk);
    a.s = a.s * pow2i(a.mk - MK) + s * pow2i(mk - MK);
    a.m = fmaxf(a.m, m);
    a.mk = MK;
}

// ---- first argmax
struct Amax {
    float best;
    int idx;
    int nan;
};

// order-independent: a thread may see its elements out of index order, so ties
// keep the lower index explicitly
__device__ __forceinline__ void amax_add(Amax& a, float x, int i)
{
    if (x > a.best || (x == a.best && i < a.idx)) { a.best = x; a.idx = i; }
    a.nan |= (x != x);
}

__device__ __forceinline__ void amax_merge(Amax& a, float best, int idx, int nan)
{
    if (best > a.best || (best == a.best && idx < a.idx)) { a.best = best; a.idx = idx; }
    a.nan |= nan;
}

// A 16-byte vector whose first element has index i0, folded into a first argmax
// that has seen only lower indices: the vector's maximum (NaN ignored), and only
// when it beats a.best the first element equal to it; a NaN anywhere makes the
// sum of the elements NaN (so does +inf with -inf, in a row the +inf already
// makes bad).  A few instructions per vector instead of a few per element.
template <int ESZ>
__device__ __forceinline__ void amax_vec(Amax& a, const uint4& v, int i0)
{
    constexpr int VEC = 16 / ESZ;
    const float m = vec_max<ESZ>(v);
    if (ESZ == 2) {
        const __nv_bfloat162 s0 = __hadd2(*reinterpret_cast<const __nv_bfloat162*>(&v.x),
                                          *reinterpret_cast<const __nv_bfloat162*>(&v.y));
        const __nv_bfloat162 s1 = __hadd2(*reinterpret_cast<const __nv_bfloat162*>(&v.z),
                                          *reinterpret_cast<const __nv_bfloat162*>(&v.w));
        const __nv_bfloat162 s2 = __hadd2(s0, s1);
        const uint32_t w = *reinterpret_cast<const uint32_t*>(&s2);
        const float t = bf16_lo(w) + bf16_hi(w);
        a.nan |= (t != t);
    } else {
        const float t = (__uint_as_float(v.x) + __uint_as_float(v.y)) + (__uint_as_float(v.z) + __uint_as_float(v.w));
        a.nan |= (t != t);
    }
    if (m > a.best) {
        float x[VEC];
        unpack<ESZ>(v, x);
        int k = VEC - 1;
#pragma unroll
        for (int e = VEC - 1; e >= 0; --e)
            if (x[e] == m) k = e;
        a.best = m;
        a.idx = i0 + k;
    }
}

// ---- block reductions over kThreads threads
__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Inclusive prefix over the 32 lanes of a warp.
__device__ __forceinline__ double warp_inclusive_scan(double x)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

template <class SYNC>
__device__ double block_sum(double v, double* sm)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    SYNC::sync();
    if (lane == 0) sm[warp] = v;
    SYNC::sync();
    double t = 0.0;
    if (threadIdx.x < 32) {
        t = lane < kWarps ? sm[lane] : 0.0;
        t = warp_sum(t);
    }
    return t;  // valid in thread 0 (warp 0)
}

// Inclusive prefix of v over the block in thread order; *total gets the block sum.
template <class SYNC>
__device__ double block_inclusive_scan(double v, double* sm, double* total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const double x = warp_inclusive_scan(v);
    SYNC::sync();
    if (lane == 31) sm[warp] = x;
    SYNC::sync();
    if (warp == 0) {
        double w = lane < kWarps ? sm[lane] : 0.0;
        w = warp_inclusive_scan(w);
        if (lane < kWarps) sm[lane] = w;
    }
    SYNC::sync();
    *total = sm[kWarps - 1];
    return (warp > 0 ? sm[warp - 1] : 0.0) + x;
}

__device__ __forceinline__ bool temperature_ok(float T)
{
    return T == 0.f || (T >= SV_TEMPERATURE_MIN && T <= FLT_MAX);
}

// k = log2(e)/T = khi + klo, khi rounded toward zero, klo > 0
__device__ __forceinline__ void split_k(float T, float* khi, float* klo)
{
    const double k = kLog2e / (double)T;
    const float hi = __double2float_rz(k);
    float lo = __double2float_rn(k - (double)hi);
    if (!(lo > 0.f)) lo = hi * 0x1p-60f;
    *khi = hi;
    *klo = lo;
}

// Residual weight max(0, p - q) of one token, or p alone (bonus draw, or the
// fallback when the residual mass is zero).  The chunk sums and the final
// in-chunk search both call this, so they see bit-identical weights.
__device__ __forceinline__ float weight_of(const SeqRec& s, bool p_only, float lt, float ld)
{
    const float p = scaled_exp(lt, s.k_hi, s.k_lo, s.mk_t) * s.inv_s_t;
    if (p_only) return p;
    const float q = scaled_exp(ld, s.k_hi, s.k_lo, s.mk_d) * s.inv_s_d;
    return fmaxf(0.f, p - q);
}

// ----------------------------------------------------------------------------- sequence tail

// Reader of one (row, chunk) partial.  raw(i) issues the load; value(raw, i,
// khi, greedy) turns it into (m, mk, s, idx-bits).  The split lets a batch of
// loads be in flight before any of them is used.
struct FloatPartials {  // Partial structs, published by a fenced ticket
    const Partial* p;
    using Raw = float4;
    __device__ __forceinline__ float4 raw(size_t i) const { return __ldcg(reinterpret_cast<const float4*>(p) + i); }
    __device__ __forceinline__ float4 value(const float4& r, size_t, float, bool) const { return r; }
};

// Everything the per-sequence finish needs: logits for the gathers, the
// small inputs, the outputs, and the workspace arrays.
struct TailArgs {
    const void* tgt;
    const void* dft;
    const int32_t* tokens;
    const float* temperature;
    const float* u_accept;
    const float* u_resample;
    int32_t* out_tokens;
    int32_t* out_n;
    double* out_log_norm;
    int32_t* out_status;
    unsigned* ticket;
    SeqRec* seq;
    const Partial* part;
    const float* gath;    // optional [B][2*gamma]: l_t[j][x_j] then l_d[j][x_j], gathered while streaming
    int gamma, V, R, nc;  // nc = partials per row
};

// Shared scratch of one sequence_tail call (one per concurrent caller).
struct TailSmem {
    double a2[kMaxRows];   // log2-normaliser of each row
    double sum[kMaxRows];  // sum relative to the integer offset
    float mk[kMaxRows];
    int arg[kMaxRows];
    int bad[kMaxRows];
    int status, n;
    SeqRec rec;  // the draw record, also stored to seq[b]
};

// Finish sequence b once every partial of its rows is written: combine the
// partials in fp64, gather log p_j(x_j) and log q_j(x_j) [FlashSpec,
// Metodologia 1, "Mecanismo"], run the log-space test at every draft position
// and take the first rejection from one warp ballot; write the accepted prefix,
// n_accepted, status, normalisers and (greedy) the extra token; store what the
// draw needs in seq[b].  Runs on NT threads numbered tid = 0..NT-1 that
// synchronise with SYNC and share `sm`.
template <int ESZ, int NT, class SYNC, class READ>
__device__ void sequence_tail(const TailArgs& a, int b, int tid, const READ& read, TailSmem& sm)
{
    double* s_a2 = sm.a2;
    double* s_sum = sm.sum;
    float* s_mk = sm.mk;
    int* s_arg = sm.arg;
    int* s_bad = sm.bad;
    int& s_status = sm.status;
    int& s_n = sm.n;

    const int lane = tid & 31, warp = tid >> 5;
    const int gamma = a.gamma, R = a.R, nc = a.nc;
    constexpr int kTailBatch = 8;
    const size_t pbase = (size_t)b * R * nc;
    const float T = a.temperature[b];
    const bool greedy = (T == 0.f);
    const bool tval = temperature_ok(T);
    const int rows_used = !tval ? 0 : (greedy ? gamma + 1 : R);
    const int32_t* tok = a.tokens + (size_t)b * gamma;
    float khi_t = 0.f, klo_t = 0.f;
    if (tval && !greedy) split_k(T, &khi_t, &klo_t);

    // the accept test's scalars, fetched first so their latency overlaps the combine
    int x_j = -1, bad_u = 0;
    double lt_j = 0.0, ld_j = 0.0, lu_j = 0.0;
    if (warp == 0 && tval && !greedy) {
        // the uniforms stand for draws of U[0, 1): anything else (NaN included)
        // is an invalid input (a greedy sequence reads none)
        if (lane < gamma) {
            const float u = a.u_accept[(size_t)b * gamma + lane];
            bad_u = !(u >= 0.f && u < 1.f);
        }
        if (lane == 0) {
            const float u = a.u_resample[b];
            bad_u |= !(u >= 0.f && u < 1.f);
        }
    }
    if (warp == 0 && lane < gamma && tval) {
        x_j = tok[lane];
        if (a.gath) {  // the streaming pass stored them: no load that waits for x_j
            lt_j = (double)__ldcg(a.gath + (size_t)b * 2 * gamma + lane);
            ld_j = (double)__ldcg(a.gath + (size_t)b * 2 * gamma + gamma + lane);
        }
        if (!greedy && x_j >= 0 && x_j < a.V) {
            const size_t V = (size_t)a.V;
            if (!a.gath) {
                lt_j = (double)load_logit<ESZ>(a.tgt, ((size_t)b * (gamma + 1) + lane) * V + x_j);
                ld_j = (double)load_logit<ESZ>(a.dft, ((size_t)b * gamma + lane) * V + x_j);
            }
            lu_j = log((double)a.u_accept[(size_t)b * gamma + lane]);
        }
    }

    // One thread per row: fold the row's partials in order.  Loads go out in
    // batches of kTailBatch before any arithmetic, so a batch costs one memory
    // latency.  Softmax rows merge (mk, s) exactly in fp64 (power-of-two scaling).
    for (int r = tid; r < rows_used; r += NT) {
        const size_t rbase = pbase + (size_t)r * nc;
        Amax A{-INFINITY, 0x7fffffff, 0};
        float m = -INFINITY, MK = 0.f;
        double S = 0.0;
        for (int c0 = 0; c0 < nc; c0 += kTailBatch) {
            typename READ::Raw raw[kTailBatch];
#pragma unroll
            for (int j = 0; j < kTailBatch; ++j)
                if (c0 + j < nc) raw[j] = read.raw(rbase + c0 + j);
#pragma unroll
            for (int j = 0; j < kTailBatch; ++j) {
                if (c0 + j >= nc) break;
                const float4 qj = read.value(raw[j], rbase + c0 + j, khi_t, greedy);
                if (greedy) {
                    amax_merge(A, qj.x, __float_as_int(qj.w), qj.z != 0.f);
                } else if (qj.x != -INFINITY) {
                    if (m == -INFINITY) {
                        m = qj.x;
                        MK = qj.y;
                        S = (double)qj.z;
                    } else if (qj.y > MK) {
                        S = S * pow2d(MK - qj.y) + (double)qj.z;
                        MK = qj.y;
                        m = fmaxf(m, qj.x);
                    } else {
                        S += (double)qj.z * pow2d(qj.y - MK);
                        m = fmaxf(m, qj.x);
                    }
                }
            }
        }
        if (greedy) {
            s_arg[r] = A.idx;
            s_bad[r] = A.nan || A.best == INFINITY || A.best == -INFINITY;
        } else {
            const bool bad = (m == -INFINITY) || (m == INFINITY) || !isfinite(S) || !(S > 0.0);
            s_bad[r] = bad;
            s_mk[r] = MK;
            s_sum[r] = S;
            s_a2[r] = bad ? NAN : (double)MK + log2(S);
        }
    }
    SYNC::sync();

    if (warp == 0) {
        int st = 0;
        if (!tval) {
            st = SV_ROW_BAD_TEMPERATURE;
        } else {
            int badtok = 0, badrow = 0;
            if (lane < gamma) badtok = (x_j < 0 || x_j >= a.V);
            for (int r = lane; r < rows_used; r += 32) badrow |= s_bad[r];
            if (__any_sync(0xffffffffu, badtok)) st |= SV_ROW_BAD_TOKEN;
            if (__any_sync(0xffffffffu, badrow)) st |= SV_ROW_BAD_LOGITS;
            if (__any_sync(0xffffffffu, bad_u)) st |= SV_ROW_BAD_UNIFORM;
        }
        int n = 0;
        if (st == 0) {
            bool acc = false;
            if (lane < gamma) {
                if (greedy) {
                    acc = (x_j == s_arg[lane]);
                } else {
                    const double Td = (double)T;
                    const double lp = lt_j / Td - s_a2[lane] * kLn2;
                    const double lq = ld_j / Td - s_a2[gamma + 1 + lane] * kLn2;
                    acc = lu_j < (lp - lq);
                }
            }
            const unsigned mask = (gamma == 32) ? 0xffffffffu : ((1u << gamma) - 1u);
            const unsigned rej = __ballot_sync(0xffffffffu, !acc) & mask;
            n = rej ? __ffs(rej) - 1 : gamma;
        }
        if (lane == 0) { s_status = st; s_n = n; }
    }
    SYNC::sync();

    const int st = s_status, n = s_n;
    int32_t* ot = a.out_tokens + (size_t)b * (gamma + 1);
    for (int j = tid; j <= gamma; j += NT) {
        int v = -1;
        if (st == 0) {
            if (j < n) v = tok[j];
            else if (j == n && greedy) v = s_arg[n];
        }
        ot[j] = v;
    }
    if (a.out_log_norm) {
        double* ln = a.out_log_norm + (size_t)b * R;
        for (int r = tid; r < R; r += NT)
            ln[r] = (tval && !greedy && !s_bad[r]) ? s_a2[r] * kLn2 : (double)NAN;
    }
    if (tid == 0) {
        a.out_n[b] = n;
        if (a.out_status) a.out_status[b] = st;
        SeqRec rec;
        rec.mode = (st != 0 || greedy) ? kModeNone : (n < gamma ? kModeResidual : kModeBonus);
        rec.n = n;
        rec.mk_t = 0.f; rec.inv_s_t = 0.f; rec.mk_d = 0.f; rec.inv_s_d = 0.f;
        rec.k_hi = 0.f; rec.k_lo = 0.f;
        if (rec.mode != kModeNone) {
            split_k(T, &rec.k_hi, &rec.k_lo);
            rec.mk_t = s_mk[n];
            rec.inv_s_t = (float)(1.0 / s_sum[n]);
            if (rec.mode == kModeResidual) {
                rec.mk_d = s_mk[gamma + 1 + n];
                rec.inv_s_d = (float)(1.0 / s_sum[gamma + 1 + n]);
            }
        }
        a.seq[b] = rec;
        sm.rec = rec;
    }
}

}  // namespace sv
