// spec_verify.cu -- B200 (sm_100a) kernels and C ABI for batched
// speculative-sampling verification.  The operation is specified in
// include/spec_verify.h; this file is the implementation.
//
// Data path (one call, no host synchronisation):
//
//   sv_rowpass   one CTA per (sequence, row, vocabulary chunk).  Streams the
//                chunk once with 128-bit non-allocating loads and keeps an
//                online (max, sum 2^(l*k - off)) pair per thread, where
//                k = log2(e)/T and `off` is an integer, so every rescale is an
//                exact power of two.  Greedy target rows keep (max, first
//                index) instead.  The CTA reduces with warp shuffles, writes a
//                16-byte partial, and takes a ticket on the sequence; the last
//                CTA of a sequence combines the partials in fp64, gathers the
//                two log-probabilities per draft position, runs the log-space
//                accept scan with one warp ballot, writes the accepted prefix
//                and, for greedy rows, the extra token.  [FlashSpec,
//                Metodologia 1: on-device test, O(1) state in V, log space,
//                temperature before the log-softmax.]
//   sv_resample  one CTA per (sequence, vocabulary chunk) of the sequences
//                that still need the extra token.  Sums the residual weights
//                max(0, p_n - q_n) (or p_gamma for the bonus token) of its
//                chunk; the last CTA of a sequence finds the chunk holding
//                u * S with a block prefix scan over chunk sums and then the
//                token inside that chunk with a second, element-level scan.
//                [Speculative Speculative Decoding, Metodologia 2: outcome =
//                accepted count + extra token; residual distribution.]
//
// Tickets: sequences complete without any spin-wait.  Every CTA increments a
// per-sequence counter after a __threadfence(); the CTA that observes the final
// count does the tail work and resets the counter to zero for the next call.
#include "spec_verify.h"

#include <cuda_runtime.h>
#include <float.h>
#include <mutex>
#include <math.h>
#include <stdint.h>

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 4;
constexpr int kMaxRows = 2 * SV_MAX_GAMMA + 1;
constexpr int kSmCount = 148;             // B200; only used to size the split of V
constexpr int kPass1ChunkBytes = 32768;   // bytes of one row streamed by one CTA
constexpr int kPass1MinChunk = 1024;      // elements
constexpr int kPass2Chunk = 8192;         // elements per residual CTA
constexpr int kPass2MinChunk = 512;
constexpr double kLn2 = 0.69314718055994530942;
constexpr double kLog2e = 1.44269504088896340736;

enum : int { kModeNone = 0, kModeResidual = 1, kModeBonus = 2 };

// Partial result of one (row, chunk).  Softmax rows: m = max logit, mk = the
// integer offset ceil(m * k_hi), s = sum of 2^(l*k - mk).  Greedy rows:
// m = max, idx = first index of the max, s != 0 if a NaN was seen.
struct __align__(16) Partial {
    float m;
    float mk;
    float s;
    int idx;
};

// What the resample kernel needs about one sequence.
struct __align__(16) SeqRec {
    int mode;
    int n;
    float mk_t;     // integer offset of target row n
    float inv_s_t;  // 1 / sum of target row n
    float mk_d;     // same for draft row n
    float inv_s_d;
    float k_hi;     // log2(e)/T split as hi + lo
    float k_lo;
};

struct Plan {
    int B, gamma, V, R, esz;
    int nc1, C1;
    int nc2, C2;
    size_t off_t1, off_t2, off_seq, off_part, off_rsum, total;
};

__host__ __device__ inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool make_plan(int B, int gamma, int V, sv_dtype dt, Plan* p)
{
    if (B < 1 || gamma < 1 || gamma > SV_MAX_GAMMA || V < 1 || V > SV_MAX_V) return false;
    if (dt != SV_DTYPE_F32 && dt != SV_DTYPE_BF16) return false;
    p->B = B;
    p->gamma = gamma;
    p->V = V;
    p->R = 2 * gamma + 1;
    p->esz = dt == SV_DTYPE_BF16 ? 2 : 4;
    const long long rows = (long long)B * p->R;
    // pass 1: ~32 KB per CTA, but at least ~2 CTAs per SM in total
    int nc1 = ceil_div((long long)V * p->esz, kPass1ChunkBytes);
    int want = ceil_div(2LL * kSmCount, rows);
    if (want > nc1) nc1 = want;
    int cap = ceil_div(V, kPass1MinChunk);
    if (nc1 > cap) nc1 = cap;
    if (nc1 < 1) nc1 = 1;
    p->C1 = ((ceil_div(V, nc1) + 7) / 8) * 8;
    p->nc1 = ceil_div(V, p->C1);
    // pass 2
    int nc2 = ceil_div(V, kPass2Chunk);
    want = ceil_div(2LL * kSmCount, B);
    if (want > nc2) nc2 = want;
    cap = ceil_div(V, kPass2MinChunk);
    if (nc2 > cap) nc2 = cap;
    if (nc2 < 1) nc2 = 1;
    p->C2 = ((ceil_div(V, nc2) + 7) / 8) * 8;
    p->nc2 = ceil_div(V, p->C2);

    size_t off = 0;
    p->off_t1 = off;
    off += sizeof(unsigned) * (size_t)B;
    p->off_t2 = off;
    off += sizeof(unsigned) * (size_t)B;
    off = align256(off);
    p->off_seq = off;
    off = align256(off + sizeof(SeqRec) * (size_t)B);
    p->off_part = off;
    off = align256(off + sizeof(Partial) * (size_t)rows * p->nc1);
    p->off_rsum = off;
    off = align256(off + sizeof(double) * (size_t)B * p->nc2);
    p->total = off;
    return true;
}

// ----------------------------------------------------------------------------- device helpers

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

// max that propagates NaN (keeps a NaN logit visible to the row-status check)
__device__ __forceinline__ float max_nan(float a, float b)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
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

// 2^(x*k - off) with k = khi + klo; -inf maps to 0, NaN stays NaN
__device__ __forceinline__ float scaled_exp(float x, float khi, float klo, float off)
{
    const float xc = max_nan(x, -FLT_MAX);
    return ex2(__fmaf_rn(xc, klo, __fmaf_rn(xc, khi, -off)));
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

// order-independent: a thread may see its elements out of index order (the
// unaligned head of a chunk is visited after the vector body), so ties keep the
// lower index explicitly
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

// ---- block reductions (kThreads threads)
__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ double block_sum(double v, double* sm)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) sm[warp] = v;
    __syncthreads();
    double t = 0.0;
    if (threadIdx.x < 32) {
        t = lane < kWarps ? sm[lane] : 0.0;
        t = warp_sum(t);
    }
    return t;  // valid in thread 0 (warp 0)
}

// Inclusive prefix of v over the block in thread order; *total gets the block sum.
__device__ double block_inclusive_scan(double v, double* sm, double* total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    double x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) sm[warp] = x;
    __syncthreads();
    if (warp == 0) {
        double w = lane < kWarps ? sm[lane] : 0.0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < kWarps) sm[lane] = w;
    }
    __syncthreads();
    *total = sm[kWarps - 1];
    return (warp > 0 ? sm[warp - 1] : 0.0) + x;
}

__device__ __forceinline__ bool temperature_ok(float T)
{
    return T == 0.f || (T >= SV_TEMPERATURE_MIN && T <= FLT_MAX);
}

__device__ __forceinline__ void split_k(float T, float* khi, float* klo)
{
    const double k = kLog2e / (double)T;
    *khi = (float)k;
    *klo = (float)(k - (double)*khi);
}

// ----------------------------------------------------------------------------- pass 1

struct Pass1Args {
    const void* tgt;
    const void* dft;
    const int32_t* tokens;
    const float* temperature;
    const float* u_accept;
    int32_t* out_tokens;
    int32_t* out_n;
    double* out_log_norm;
    int32_t* out_status;
    unsigned* ticket;
    SeqRec* seq;
    Partial* part;
    int gamma, V, R, nc1, C1;
};

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
    for (; i + (kUnroll - 1) * kThreads < nvec; i += kUnroll * kThreads) {
        uint4 r[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) r[u] = ld_stream(vp + i + u * kThreads);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            float x[VEC];
            unpack<ESZ>(r[u], x);
            if (GREEDY) {
                const int e0 = vbase + (i + u * kThreads) * VEC;
#pragma unroll
                for (int e = 0; e < VEC; ++e) amax_add(A, x[e], e0 + e);
            } else {
                lse_add<VEC>(L, x, khi, klo);
            }
        }
    }
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

template <int ESZ>
__device__ void sequence_tail(const Pass1Args& a, int b, float T, bool greedy)
{
    __shared__ double s_a2[kMaxRows];   // log2-normaliser of each row
    __shared__ double s_sum[kMaxRows];  // sum relative to the integer offset
    __shared__ float s_mk[kMaxRows];
    __shared__ int s_arg[kMaxRows];
    __shared__ int s_bad[kMaxRows];
    __shared__ int s_status, s_n;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gamma = a.gamma, R = a.R, nc = a.nc1;
    const bool tval = temperature_ok(T);
    const int rows_used = !tval ? 0 : (greedy ? gamma + 1 : R);
    const Partial* pp = a.part + (size_t)b * R * nc;

    for (int r = warp; r < rows_used; r += kWarps) {
        if (greedy) {
            Amax A{-INFINITY, 0x7fffffff, 0};
            for (int c = lane; c < nc; c += 32) {
                const float4 q = __ldcg(reinterpret_cast<const float4*>(pp + (size_t)r * nc + c));
                amax_merge(A, q.x, __float_as_int(q.w), q.z != 0.f);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ob = __shfl_xor_sync(0xffffffffu, A.best, o);
                const int oi = __shfl_xor_sync(0xffffffffu, A.idx, o);
                const int on = __shfl_xor_sync(0xffffffffu, A.nan, o);
                amax_merge(A, ob, oi, on);
            }
            if (lane == 0) {
                s_arg[r] = A.idx;
                s_bad[r] = A.nan || A.best == INFINITY || A.best == -INFINITY;
            }
        } else {
            float m = -INFINITY, mk = -INFINITY;
            for (int c = lane; c < nc; c += 32) {
                const float4 q = __ldcg(reinterpret_cast<const float4*>(pp + (size_t)r * nc + c));
                if (q.x != -INFINITY) { m = fmaxf(m, q.x); mk = fmaxf(mk, q.y); }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o));
            }
            double s = 0.0;
            if (m != -INFINITY && m != INFINITY) {
                for (int c = lane; c < nc; c += 32) {
                    const float4 q = __ldcg(reinterpret_cast<const float4*>(pp + (size_t)r * nc + c));
                    if (q.x != -INFINITY) s += ldexp((double)q.z, (int)(q.y - mk));
                }
            }
            s = warp_sum(s);
            if (lane == 0) {
                const bool bad = (m == -INFINITY) || (m == INFINITY) || !isfinite(s) || !(s > 0.0);
                s_bad[r] = bad;
                s_mk[r] = mk;
                s_sum[r] = s;
                s_a2[r] = bad ? NAN : (double)mk + log2(s);
            }
        }
    }
    __syncthreads();

    const int32_t* tok = a.tokens + (size_t)b * gamma;
    if (warp == 0) {
        int st = 0;
        if (!tval) {
            st = SV_ROW_BAD_TEMPERATURE;
        } else {
            int badtok = 0, badrow = 0;
            if (lane < gamma) { const int x = tok[lane]; badtok = (x < 0 || x >= a.V); }
            for (int r = lane; r < rows_used; r += 32) badrow |= s_bad[r];
            if (__any_sync(0xffffffffu, badtok)) st |= SV_ROW_BAD_TOKEN;
            if (__any_sync(0xffffffffu, badrow)) st |= SV_ROW_BAD_LOGITS;
        }
        int n = 0;
        if (st == 0) {
            bool acc = false;
            if (lane < gamma) {
                const int x = tok[lane];
                if (greedy) {
                    acc = (x == s_arg[lane]);
                } else {
                    const size_t V = (size_t)a.V;
                    const double lt = (double)load_logit<ESZ>(a.tgt, ((size_t)b * (gamma + 1) + lane) * V + x);
                    const double ld = (double)load_logit<ESZ>(a.dft, ((size_t)b * gamma + lane) * V + x);
                    const double Td = (double)T;
                    const double lp = lt / Td - s_a2[lane] * kLn2;
                    const double lq = ld / Td - s_a2[gamma + 1 + lane] * kLn2;
                    const double lu = log((double)a.u_accept[(size_t)b * gamma + lane]);
                    acc = lu < (lp - lq);
                }
            }
            const unsigned rej = __ballot_sync(0xffffffffu, !acc) & ((gamma == 32) ? 0xffffffffu : ((1u << gamma) - 1u));
            n = rej ? __ffs(rej) - 1 : gamma;
        }
        if (lane == 0) { s_status = st; s_n = n; }
    }
    __syncthreads();

    const int st = s_status, n = s_n;
    int32_t* ot = a.out_tokens + (size_t)b * (gamma + 1);
    for (int j = threadIdx.x; j <= gamma; j += kThreads) {
        int v = -1;
        if (st == 0) {
            if (j < n) v = tok[j];
            else if (j == n && greedy) v = s_arg[n];
        }
        ot[j] = v;
    }
    if (a.out_log_norm) {
        double* ln = a.out_log_norm + (size_t)b * R;
        for (int r = threadIdx.x; r < R; r += kThreads)
            ln[r] = (tval && !greedy && !s_bad[r]) ? s_a2[r] * kLn2 : (double)NAN;
    }
    if (threadIdx.x == 0) {
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
        a.ticket[b] = 0u;  // every CTA of this sequence has arrived: ready for the next call
    }
}

template <int ESZ>
__global__ void __launch_bounds__(kThreads) sv_rowpass(Pass1Args a)
{
    __shared__ float s_red[3 * kWarps];
    __shared__ int s_last;

    const int c = blockIdx.x % a.nc1;
    const int rr = blockIdx.x / a.nc1;
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
        const int v0 = c * a.C1;
        const int v1 = min(a.V, v0 + a.C1);
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        Partial out;
        if (greedy) {
            Lse L;
            Amax A{-INFINITY, 0x7fffffff, 0};
            scan_chunk<ESZ, true>(rowp, v0, v1, 0.f, 0.f, L, A);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ob = __shfl_xor_sync(0xffffffffu, A.best, o);
                const int oi = __shfl_xor_sync(0xffffffffu, A.idx, o);
                const int on = __shfl_xor_sync(0xffffffffu, A.nan, o);
                amax_merge(A, ob, oi, on);
            }
            if (lane == 0) {
                s_red[warp] = A.best;
                s_red[kWarps + warp] = __int_as_float(A.idx);
                s_red[2 * kWarps + warp] = (float)A.nan;
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                Amax F{-INFINITY, 0x7fffffff, 0};
                for (int w = 0; w < kWarps; ++w)
                    amax_merge(F, s_red[w], __float_as_int(s_red[kWarps + w]), s_red[2 * kWarps + w] != 0.f);
                out.m = F.best;
                out.mk = 0.f;
                out.s = (float)F.nan;
                out.idx = F.idx;
            }
        } else {
            float khi, klo;
            split_k(T, &khi, &klo);
            Lse L;
            lse_init(L);
            Amax A;
            scan_chunk<ESZ, false>(rowp, v0, v1, khi, klo, L, A);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float om = __shfl_xor_sync(0xffffffffu, L.m, o);
                const float omk = __shfl_xor_sync(0xffffffffu, L.mk, o);
                const float os = __shfl_xor_sync(0xffffffffu, L.s, o);
                lse_merge(L, om, omk, os);
            }
            if (lane == 0) {
                s_red[warp] = L.m;
                s_red[kWarps + warp] = L.mk;
                s_red[2 * kWarps + warp] = L.s;
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                Lse F;
                lse_init(F);
                for (int w = 0; w < kWarps; ++w) lse_merge(F, s_red[w], s_red[kWarps + w], s_red[2 * kWarps + w]);
                out.m = F.m;
                out.mk = F.mk;
                out.s = F.s;
                out.idx = 0;
            }
        }
        if (threadIdx.x == 0) a.part[((size_t)b * a.R + r) * a.nc1 + c] = out;
    }

    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&a.ticket[b], 1u);
        s_last = (prev == (unsigned)(a.R * a.nc1 - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    sequence_tail<ESZ>(a, b, T, greedy);
}

// ----------------------------------------------------------------------------- pass 2

struct Pass2Args {
    const void* tgt;
    const void* dft;
    const float* u_resample;
    int32_t* out_tokens;
    int32_t* out_status;
    unsigned* ticket;
    const SeqRec* seq;
    double* rsum;
    int gamma, V, nc2, C2;
};

// Residual weight max(0, p - q) of one token, or p alone (bonus draw, or the
// fallback when the residual mass is zero).  Both the chunk sums and the final
// in-chunk search call this, so they see bit-identical weights.
__device__ __forceinline__ float weight_of(const SeqRec& s, bool p_only, float lt, float ld)
{
    const float p = scaled_exp(lt, s.k_hi, s.k_lo, s.mk_t) * s.inv_s_t;
    if (p_only) return p;
    const float q = scaled_exp(ld, s.k_hi, s.k_lo, s.mk_d) * s.inv_s_d;
    return fmaxf(0.f, p - q);
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
            float part = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) part += weight_of(s, p_only, xt[e], p_only ? 0.f : xd[e]);
            acc += (double)part;
        }
        done = nvec * VEC;
    }
    for (int e = done + tid; e < n; e += kThreads) {
        const float lt = load_logit<ESZ>(trow, (size_t)(v0 + e));
        const float ld = p_only ? 0.f : load_logit<ESZ>(drow, (size_t)(v0 + e));
        acc += (double)weight_of(s, p_only, lt, ld);
    }
    return block_sum(acc, sm);
}

// Inverse CDF over the sequence's weights, given the per-chunk sums in rs[]:
// the smallest token k with running sum C_k > u * S; if rounding leaves none,
// the last token with a positive weight.
template <int ESZ>
__device__ void sequence_draw(const Pass2Args& a, int b, const SeqRec& s, const unsigned char* trow,
                              const unsigned char* drow)
{
    __shared__ double s_scan[kWarps];
    __shared__ double s_bcast;
    __shared__ int s_found, s_lastpos;

    const int tid = threadIdx.x;
    const int nc = a.nc2, C = a.C2, V = a.V;
    double* rs = a.rsum + (size_t)b * nc;
    bool p_only = (s.mode == kModeBonus);

    // total mass, in the same tile-scan order that the chunk search below uses
    double S = 0.0;
    for (int c0 = 0; c0 < nc; c0 += kThreads) {
        double tot;
        block_inclusive_scan((c0 + tid < nc) ? __ldcg(rs + c0 + tid) : 0.0, s_scan, &tot);
        S += tot;
    }
    int flag = 0;
    if (!(S > 0.0) && s.mode == kModeResidual) {
        // the residual vanished (p == q up to rounding): draw from p_n instead
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
            block_inclusive_scan((c0 + tid < nc) ? rs[c0 + tid] : 0.0, s_scan, &tot);
            S += tot;
        }
    }
    const double target = (double)a.u_resample[b] * S;

    // 1) the chunk c* holding the target: first chunk whose inclusive prefix > target
    if (tid == 0) { s_found = 0x7fffffff; s_lastpos = -1; s_bcast = 0.0; }
    __syncthreads();
    double carry = 0.0;
    int cstar = -1;
    for (int c0 = 0; c0 < nc; c0 += kThreads) {
        const int c = c0 + tid;
        const double v = (c < nc) ? __ldcg(rs + c) : 0.0;
        double tot;
        const double incl = carry + block_inclusive_scan(v, s_scan, &tot);
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
        double c = run + block_inclusive_scan(loc, s_scan, &tot) - loc;
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
        a.out_tokens[(size_t)b * (a.gamma + 1) + s.n] = k;
        if (flag && a.out_status) a.out_status[b] |= flag;
        a.ticket[b] = 0u;
    }
}

template <int ESZ>
__global__ void __launch_bounds__(kThreads) sv_resample(Pass2Args a)
{
    __shared__ double s_red[kWarps];
    __shared__ int s_last;

    const int c = blockIdx.x % a.nc2;
    const int b = blockIdx.x / a.nc2;
    const SeqRec s = a.seq[b];
    if (s.mode == kModeNone) return;

    const size_t V = (size_t)a.V;
    const unsigned char* trow = static_cast<const unsigned char*>(a.tgt) +
                                ((size_t)b * (a.gamma + 1) + s.n) * V * ESZ;
    const unsigned char* drow = s.mode == kModeResidual
                                    ? static_cast<const unsigned char*>(a.dft) + ((size_t)b * a.gamma + s.n) * V * ESZ
                                    : nullptr;
    const int v0 = c * a.C2;
    const int v1 = min(a.V, v0 + a.C2);
    const double cs = chunk_weight_sum<ESZ>(trow, drow, s, s.mode == kModeBonus, v0, v1, s_red);
    if (threadIdx.x == 0) {
        a.rsum[(size_t)b * a.nc2 + c] = cs;
        __threadfence();
        const unsigned prev = atomicAdd(&a.ticket[b], 1u);
        s_last = (prev == (unsigned)(a.nc2 - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    sequence_draw<ESZ>(a, b, s, trow, drow);
}

template <int ESZ>
cudaError_t launch(const Plan& p, const void* tgt, const void* dft, const int32_t* tokens,
                   const float* temperature, const float* u_acc, const float* u_res, int32_t* out_tokens,
                   int32_t* out_n, double* out_ln, int32_t* out_st, unsigned char* ws, cudaStream_t st)
{
    Pass1Args a1;
    a1.tgt = tgt;
    a1.dft = dft;
    a1.tokens = tokens;
    a1.temperature = temperature;
    a1.u_accept = u_acc;
    a1.out_tokens = out_tokens;
    a1.out_n = out_n;
    a1.out_log_norm = out_ln;
    a1.out_status = out_st;
    a1.ticket = reinterpret_cast<unsigned*>(ws + p.off_t1);
    a1.seq = reinterpret_cast<SeqRec*>(ws + p.off_seq);
    a1.part = reinterpret_cast<Partial*>(ws + p.off_part);
    a1.gamma = p.gamma;
    a1.V = p.V;
    a1.R = p.R;
    a1.nc1 = p.nc1;
    a1.C1 = p.C1;
    const long long g1 = (long long)p.B * p.R * p.nc1;
    if (g1 > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    sv_rowpass<ESZ><<<(unsigned)g1, kThreads, 0, st>>>(a1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    Pass2Args a2;
    a2.tgt = tgt;
    a2.dft = dft;
    a2.u_resample = u_res;
    a2.out_tokens = out_tokens;
    a2.out_status = out_st;
    a2.ticket = reinterpret_cast<unsigned*>(ws + p.off_t2);
    a2.seq = reinterpret_cast<const SeqRec*>(ws + p.off_seq);
    a2.rsum = reinterpret_cast<double*>(ws + p.off_rsum);
    a2.gamma = p.gamma;
    a2.V = p.V;
    a2.nc2 = p.nc2;
    a2.C2 = p.C2;
    const long long g2 = (long long)p.B * p.nc2;
    if (g2 > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    sv_resample<ESZ><<<(unsigned)g2, kThreads, 0, st>>>(a2);
    return cudaGetLastError();
}

inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace

// ============================================================================= C ABI

extern "C" size_t spec_verify_workspace_size(int B, int gamma, int V, sv_dtype dt)
{
    Plan p;
    return make_plan(B, gamma, V, dt, &p) ? p.total : 0;
}

extern "C" sv_status spec_verify_workspace_init(void* workspace, size_t workspace_bytes,
                                                struct CUstream_st* stream)
{
    if (!workspace && workspace_bytes) return SV_ERR_INVALID_ARG;
    if (!workspace_bytes) return SV_OK;
    return cudaMemsetAsync(workspace, 0, workspace_bytes, (cudaStream_t)stream) == cudaSuccess ? SV_OK
                                                                                               : SV_ERR_CUDA;
}

extern "C" sv_status spec_verify(const void* target_logits, const void* draft_logits, sv_dtype dt,
                                 const int32_t* draft_tokens, const float* temperature,
                                 const float* u_accept, const float* u_resample, int32_t* out_tokens,
                                 int32_t* out_n_accepted, int B, int gamma, int V, void* workspace,
                                 size_t workspace_bytes, double* out_log_norm, int32_t* out_row_status,
                                 struct CUstream_st* stream)
{
    if (dt != SV_DTYPE_F32 && dt != SV_DTYPE_BF16) return SV_ERR_UNSUPPORTED_DTYPE;
    Plan p;
    if (!make_plan(B, gamma, V, dt, &p)) return SV_ERR_INVALID_ARG;
    if (!target_logits || !draft_logits || !draft_tokens || !temperature || !u_accept || !u_resample ||
        !out_tokens || !out_n_accepted || !workspace)
        return SV_ERR_INVALID_ARG;
    if (!aligned(target_logits, 16) || !aligned(draft_logits, 16) || !aligned(draft_tokens, 4) ||
        !aligned(temperature, 4) || !aligned(u_accept, 4) || !aligned(u_resample, 4) || !aligned(out_tokens, 4) ||
        !aligned(out_n_accepted, 4) || !aligned(workspace, 256) || !aligned(out_log_norm, 8) ||
        !aligned(out_row_status, 4))
        return SV_ERR_MISALIGNED;
    if (workspace_bytes < p.total) return SV_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const cudaError_t e =
        dt == SV_DTYPE_BF16
            ? launch<2>(p, target_logits, draft_logits, draft_tokens, temperature, u_accept, u_resample, out_tokens,
                        out_n_accepted, out_log_norm, out_row_status, ws, st)
            : launch<4>(p, target_logits, draft_logits, draft_tokens, temperature, u_accept, u_resample, out_tokens,
                        out_n_accepted, out_log_norm, out_row_status, ws, st);
    return e == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}

extern "C" const char* spec_verify_status_string(sv_status s)
{
    switch (s) {
    case SV_OK: return "ok";
    case SV_ERR_INVALID_ARG: return "invalid argument (size, null pointer or enum)";
    case SV_ERR_UNSUPPORTED_DTYPE: return "unsupported logits dtype";
    case SV_ERR_MISALIGNED: return "misaligned pointer (logits need 16 bytes, workspace 256)";
    case SV_ERR_WORKSPACE_TOO_SMALL: return "workspace smaller than spec_verify_workspace_size()";
    case SV_ERR_CUDA: return "CUDA launch or runtime error";
    }
    return "unknown status";
}

// ============================================================================= no-allocation variant
//
// For callers that cannot allocate device memory (see spec_verify_noalloc in the
// header): the workspace is this fixed array, one per GPU for the life of the
// process.  Host code must not pass the symbol itself to a kernel (on the host it
// names a stand-in, not device memory); its device address is looked up once per
// device below.

static __device__ __align__(256) unsigned char sv_noalloc_scratch[SV_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of sv_noalloc_scratch on the current device (first use per device
// does the lookup).  Returns nullptr on a CUDA error.
void* noalloc_scratch_address()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, sv_noalloc_scratch) != cudaSuccess || !p) return nullptr;
        g_noalloc_ptr[dev] = p;
    }
    return g_noalloc_ptr[dev];
}
}  // namespace

extern "C" sv_status spec_verify_noalloc(const void* target_logits, const void* draft_logits, sv_dtype dt,
                                         const int32_t* draft_tokens, const float* temperature,
                                         const float* u_accept, const float* u_resample, int32_t* out_tokens,
                                         int32_t* out_n_accepted, int B, int gamma, int V, double* out_log_norm,
                                         int32_t* out_row_status, struct CUstream_st* stream)
{
    if (dt != SV_DTYPE_F32 && dt != SV_DTYPE_BF16) return SV_ERR_UNSUPPORTED_DTYPE;
    Plan p;
    if (!make_plan(B, gamma, V, dt, &p)) return SV_ERR_INVALID_ARG;
    if (!target_logits || !draft_logits || !draft_tokens || !temperature || !u_accept || !u_resample ||
        !out_tokens || !out_n_accepted)
        return SV_ERR_INVALID_ARG;
    if (!aligned(target_logits, 16) || !aligned(draft_logits, 16) || !aligned(draft_tokens, 4) ||
        !aligned(temperature, 4) || !aligned(u_accept, 4) || !aligned(u_resample, 4) || !aligned(out_tokens, 4) ||
        !aligned(out_n_accepted, 4) || !aligned(out_log_norm, 8) || !aligned(out_row_status, 4))
        return SV_ERR_MISALIGNED;
    if (p.total > SV_NOALLOC_SCRATCH_BYTES) return SV_ERR_WORKSPACE_TOO_SMALL;
    unsigned char* ws = static_cast<unsigned char*>(noalloc_scratch_address());
    if (!ws) return SV_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    // the completion counters must start at zero; the rest is overwritten before use
    if (cudaMemsetAsync(ws, 0, p.off_seq, st) != cudaSuccess) return SV_ERR_CUDA;
    const cudaError_t e =
        dt == SV_DTYPE_BF16
            ? launch<2>(p, target_logits, draft_logits, draft_tokens, temperature, u_accept, u_resample, out_tokens,
                        out_n_accepted, out_log_norm, out_row_status, ws, st)
            : launch<4>(p, target_logits, draft_logits, draft_tokens, temperature, u_accept, u_resample, out_tokens,
                        out_n_accepted, out_log_norm, out_row_status, ws, st);
    return e == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}
