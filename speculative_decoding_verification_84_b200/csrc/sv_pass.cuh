// sv_pass.cuh -- the streaming path for rows that are 16-byte aligned and at
// least 4 KB: two kernels, the second a programmatic dependent of the first.
//
//   sv_stream  every warp of a resident grid takes one contiguous span of the
//              row stream and walks it on its own (no barrier, no atomic, no
//              wait), 4 vectors per lane per batch, keeping a lagging-offset
//              log-sum-exp of l/T (sv_common.cuh) or the first argmax (T = 0).
//              Where its span crosses a row boundary the warp reduces with
//              shuffles and writes one Partial for that row segment; the warp
//              holding a row's draft token keeps the logit l[x_j] for the accept
//              test from its registers.  The next row's temperature and token are
//              fetched one segment ahead, so no load waits on another.
//              The rows are streamed by draft position, last position first and
//              position 0 last: the rows a draw most often reads again (the
//              first rejection is most often early) are the last ones streamed
//              and are still in L2 when sv_draw reads them; rows streamed earlier
//              are loaded with an L2 evict-first hint so they do not push them out.
//   sv_draw    one thread-block cluster per sequence b (clusters loop over the
//              sequences).  Every CTA of the cluster finishes b on its own --
//              fp64 combine of the partials (every load of the finish in
//              flight at once), the log-space accept test [FlashSpec,
//              Metodologia 1] with the first rejection from one ballot -- so no
//              CTA waits for another to learn the outcome.  The CTAs then split
//              the draw rows (residual max(0, p_n - q_n), or p_gamma for the bonus
//              token) [Speculative Speculative Decoding, Metodologia 2, "Conceito
//              Central"; Desafios 2, "Amostragem Saguaro"] into tiles of 32
//              vectors, one fp32 weight sum per tile in the CTA's own shared
//              memory, and send their totals to every CTA through distributed
//              shared memory.  After one cluster barrier each CTA knows S and
//              which CTA's range holds u * S; that CTA draws the token by inverse
//              CDF over its own tile sums, then inside the tile.
// sv_stream triggers its dependents at entry, so sv_draw's CTAs start as
// sv_stream's leave; they fetch their sequence's inputs, take the logarithms and
// reciprocals those alone decide, and then wait (griddepcontrol.wait) for all of
// sv_stream before reading its partials.
// Nothing is carried between calls: every slot a call reads, it wrote.
#pragma once

#include "sv_common.cuh"
#include "sv_generic.cuh"

#include <cooperative_groups.h>

namespace sv {

namespace cg = cooperative_groups;

constexpr int kPassThreads = 256;                  // = kThreads: block reductions apply
constexpr int kStreamVec = 4;                      // 16-byte vectors per lane per sv_stream batch
constexpr int kStreamSlots = 32;                   // partial slots per row (spans >= nq / 31 vectors)
constexpr int kStreamSpanMin = 128;                // shortest span of a warp (vectors)
constexpr int kMaxCluster = 8;                     // sv_draw cluster size limit (portable)
constexpr int kTileSmem = 4096;                    // a CTA keeps up to this many tile sums in shared memory
constexpr int kTileVecs = 32;                      // vectors per tile (one per lane)
constexpr int kTileU = 4;                          // tiles per warp per batch in sv_draw
constexpr int kStreamMinRowBytes = 4096;           // shorter rows take the generic path
constexpr int kDrawQ = 16;                         // tile sums per lane per draw block

static_assert(kPassThreads == kThreads, "block reductions assume kThreads threads");

struct PassArgs {
    TailArgs t;              // t.nc = kStreamSlots
    Partial* part;           // [B][R][kStreamSlots]; the slots no span fills hold empty partials
    float* gath;             // [B][2*gamma] the accept test's logits, written by sv_stream
    float* tsum;             // [B][NT2] weight sum of each tile (rows of more than kTileSmem tiles)
    const float* u_resample;
    long long nq;            // 16-byte vectors per row
    long long S;             // vectors per warp span (sv_stream)
    long long evict_rows;    // stream rows [0, evict_rows) load with an L2 evict-first hint
    int NT2;                 // tiles per row
    int B;
};

template <int ESZ>
__device__ __forceinline__ const unsigned char* row_ptr(const TailArgs& t, int b, int r)
{
    const size_t V = (size_t)t.V;
    return r <= t.gamma
               ? static_cast<const unsigned char*>(t.tgt) + ((size_t)b * (t.gamma + 1) + r) * V * ESZ
               : static_cast<const unsigned char*>(t.dft) + ((size_t)b * t.gamma + (r - t.gamma - 1)) * V * ESZ;
}

template <int ESZ>
__device__ __forceinline__ uint4 neg_inf_vec()
{
    const unsigned w = ESZ == 2 ? 0xff80ff80u : 0xff800000u;
    return make_uint4(w, w, w, w);
}

// ----------------------------------------------------------------------------- sv_stream

// Stream order of the rows: the bonus rows (target row gamma) of every sequence
// first, then for j = gamma-1 down to 0 the pairs (target row j, draft row j) of
// every sequence.  Stream row ro -> sequence b and row r of it (r > gamma: draft).
__device__ __forceinline__ void stream_row(int gamma, int B, long long ro, int& b, int& r)
{
    if (ro < B) {
        b = (int)ro;
        r = gamma;
        return;
    }
    const long long k = ro - B;
    const int j = gamma - 1 - (int)(k / (2LL * B));
    const long long m = k - (long long)(gamma - 1 - j) * 2LL * B;
    b = (int)(m >> 1);
    r = (m & 1) ? gamma + 1 + j : j;
}

// the draft position a row tests (-1 for the bonus row)
__device__ __forceinline__ int row_position(int gamma, int r)
{
    return r < gamma ? r : (r > gamma ? r - gamma - 1 : -1);
}

template <bool EVF>
__device__ __forceinline__ uint4 ld_row(const uint4* p, unsigned long long pol)
{
    if (!EVF) return ld_stream(p);
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

// element e of a 16-byte vector
template <int ESZ>
__device__ __forceinline__ float vec_elem(const uint4& v, int e)
{
    const int wi = ESZ == 2 ? (e >> 1) : e;
    const unsigned w = wi == 0 ? v.x : (wi == 1 ? v.y : (wi == 2 ? v.z : v.w));
    if (ESZ == 4) return __uint_as_float(w);
    return (e & 1) ? bf16_hi(w) : bf16_lo(w);
}

// The exact form of a segment's sum, for a segment whose lagging offset was off
// (sum outside [2^-40, 2^100), or not finite): the warp's maximum first, then the
// sum of 2^(l*k - ceil(max*k_hi)).  Re-reads the segment (mostly from L2).
template <int ESZ>
__device__ __noinline__ float2 stream_exact(const uint4* p, int n, float khi, float klo, float mk)
{
    const int lane = threadIdx.x & 31;
    float vm = -INFINITY;
    for (int i = lane; i < n; i += 32) vm = fmaxf(vm, vec_max<ESZ>(ld_stream(p + i)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, o));
    if (vm > -INFINITY && vm < INFINITY) mk = ceilf(__fmul_rn(vm, khi));
    unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
    for (int i = lane; i < n; i += 32) {
        const uint4 v = ld_stream(p + i);
        lazy_exps_add<ESZ, 1>(acc, &v, khi, klo, mk);
    }
    return make_float2(mk, lazy_warp_sum(acc));
}

// One softmax segment [p, p + n) against the carried offset mk: the warp's
// (offset, sum); *gval gets element ex of vector qx (qx < 0: none), in lane qx & 31.
template <int ESZ, bool EVF>
__device__ __forceinline__ float2 stream_softmax(const uint4* p, int n, float khi, float klo, float& mk, int qx,
                                                 int ex, float* gval, unsigned long long pol)
{
    constexpr int CV = 32 * kStreamVec;
    const int lane = threadIdx.x & 31;
    const int kb = qx >= 0 ? qx / CV : -1;
    const int ux = qx >= 0 ? (qx % CV) >> 5 : 0;
    const int lx = qx & 31;
    unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
    int jb = 0;
    for (int j0 = 0; j0 < n; j0 += CV, ++jb) {
        uint4 v[kStreamVec];
        if (j0 + CV <= n) {
#pragma unroll
            for (int u = 0; u < kStreamVec; ++u) v[u] = ld_row<EVF>(p + j0 + u * 32 + lane, pol);
        } else {
#pragma unroll
            for (int u = 0; u < kStreamVec; ++u) {
                const int i = j0 + u * 32 + lane;
                v[u] = i < n ? ld_row<EVF>(p + i, pol) : neg_inf_vec<ESZ>();
            }
        }
        if (jb == kb && lane == lx) {
            uint4 t = v[0];
#pragma unroll
            for (int u = 1; u < kStreamVec; ++u)
                if (u == ux) t = v[u];
            *gval = vec_elem<ESZ>(t, ex);
        }
        lazy_exps_add<ESZ, kStreamVec>(acc, v, khi, klo, mk);
    }
    const float s = lazy_warp_sum(acc);
    if (s >= 0x1p-40f && s < 0x1p100f) return make_float2(mk, s);
    const float2 r = stream_exact<ESZ>(p, n, khi, klo, mk);
    mk = r.x;
    return r;
}

// One row segment [q0, q0 + n) of row (b, r) with temperature T and draft token
// x (-1 for the bonus row): the warp's Partial, and l[x] for the accept test.
template <int ESZ>
__device__ __forceinline__ void stream_segment(const PassArgs& g, int b, int r, float T, int x, long long q0, int n,
                                               Partial* dst, float& mk, bool evf, unsigned long long pol)
{
    constexpr int VEC = 16 / ESZ;
    constexpr int kStep = 32 * kStreamVec;
    const TailArgs& a = g.t;
    const int lane = threadIdx.x & 31;
    if (!temperature_ok(T) || (T == 0.f && r > a.gamma)) return;  // a row the finish will not read
    const uint4* p = reinterpret_cast<const uint4*>(row_ptr<ESZ>(a, b, r)) + q0;
    if (T == 0.f) {
        Amax A{-INFINITY, 0x7fffffff, 0};
        const int e0 = (int)(q0 * VEC);
        for (int j0 = 0; j0 < n; j0 += kStep) {
            uint4 v[kStreamVec];
#pragma unroll
            for (int u = 0; u < kStreamVec; ++u) {
                const int i = j0 + u * 32 + lane;
                v[u] = i < n ? ld_stream(p + i) : neg_inf_vec<ESZ>();
            }
            // a lane meets its vectors in increasing index order; fill vectors
            // (-inf past the segment) never beat a real maximum
#pragma unroll
            for (int u = 0; u < kStreamVec; ++u) amax_vec<ESZ>(A, v[u], e0 + (j0 + u * 32 + lane) * VEC);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, A.best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, A.idx, o);
            const int on = __shfl_xor_sync(0xffffffffu, A.nan, o);
            amax_merge(A, ob, oi, on);
        }
        if (lane == 0) *dst = Partial{A.best, 0.f, (float)A.nan, A.idx};
        return;
    }
    float khi, klo;
    split_k(T, &khi, &klo);
    int qx = -1, ex = 0;
    if (x >= 0 && x < a.V) {
        const long long q = (long long)(x / VEC) - q0;
        if (q >= 0 && q < n) {
            qx = (int)q;
            ex = x % VEC;
        }
    }
    float gval = 0.f;
    const float2 ms = evf ? stream_softmax<ESZ, true>(p, n, khi, klo, mk, qx, ex, &gval, pol)
                          : stream_softmax<ESZ, false>(p, n, khi, klo, mk, qx, ex, &gval, pol);
    // an all -inf segment (sum 0) is an empty partial; m only marks presence
    if (lane == 0) *dst = Partial{ms.y != 0.f ? 0.f : -INFINITY, ms.x, ms.y, 0};
    if (qx >= 0 && lane == (qx & 31)) {
        const int j = row_position(a.gamma, r);
        g.gath[(size_t)b * 2 * a.gamma + (r < a.gamma ? j : a.gamma + j)] = gval;
    }
}

template <int ESZ>
__global__ void __launch_bounds__(kPassThreads, 4) sv_stream(const __grid_constant__ PassArgs g)
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // sv_draw may be scheduled
    const TailArgs& a = g.t;
    const int lane = threadIdx.x & 31;
    const long long w = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const long long NQ = (long long)g.B * a.R * g.nq;
    long long cur = w * g.S;
    const long long v1 = min(cur + g.S, NQ);
    if (cur >= v1) return;
    unsigned long long pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    float mk = 0.f;  // lagging offset, carried across segments
    long long ro = cur / g.nq;
    int b, r;
    stream_row(a.gamma, g.B, ro, b, r);
    float T = __ldg(a.temperature + b);
    int jp = row_position(a.gamma, r);
    int x = jp >= 0 ? __ldg(a.tokens + (size_t)b * a.gamma + jp) : -1;
    while (cur < v1) {
        const long long rend = (ro + 1) * g.nq;
        const long long pend = min(v1, rend);
        // the next row's temperature and token, one segment ahead
        int bn = 0, rn = 0, xn = -1;
        float Tn = 0.f;
        if (pend < v1) {
            stream_row(a.gamma, g.B, ro + 1, bn, rn);
            Tn = __ldg(a.temperature + bn);
            const int jn = row_position(a.gamma, rn);
            if (jn >= 0) xn = __ldg(a.tokens + (size_t)bn * a.gamma + jn);
        }
        // spans s0 .. w meet the row so far: this segment is slot w - s0
        const int slot = (int)(w - (ro * g.nq) / g.S);
        Partial* prow = g.part + ((size_t)b * a.R + r) * kStreamSlots;
        stream_segment<ESZ>(g, b, r, T, x, cur - ro * g.nq, (int)(pend - cur), prow + slot, mk, ro < g.evict_rows,
                            pol);
        // the span that ends the row marks the row's remaining slots empty, so the
        // finish reads a fixed kStreamSlots slots per row
        if (pend == rend)
            for (int k = slot + 1 + lane; k < kStreamSlots; k += 32) prow[k] = Partial{-INFINITY, 0.f, 0.f, 0x7fffffff};
        cur = pend;
        ++ro;
        b = bn;
        r = rn;
        T = Tn;
        x = xn;
    }
}

// ----------------------------------------------------------------------------- sv_draw

// A block of up to 32*kDrawQ tile sums: lane l holds tiles s0 + l*kDrawQ + q.
struct TileBlock {
    float v[kDrawQ];
    double ls;    // the lane's sum, in tile order
    double incl;  // inclusive prefix of ls over lanes
};

// w is either this CTA's shared memory (smem) or global memory written by other
// CTAs of the cluster (read at L2).
__device__ __forceinline__ void load_tile_block(TileBlock& tb, const float* w, int n, int s0, bool smem)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int q = 0; q < kDrawQ; ++q) {
        const int idx = s0 + lane * kDrawQ + q;
        tb.v[q] = idx < n ? (smem ? w[idx] : __ldcg(w + idx)) : 0.f;
    }
    double t[kDrawQ / 2];
#pragma unroll
    for (int q = 0; q < kDrawQ / 2; ++q) t[q] = (double)tb.v[2 * q] + (double)tb.v[2 * q + 1];
#pragma unroll
    for (int w = kDrawQ / 4; w >= 1; w >>= 1)
#pragma unroll
        for (int q = 0; q < w; ++q) t[q] += t[q + w];
    tb.ls = t[0];
    tb.incl = warp_inclusive_scan(tb.ls);
}

// First tile of the block whose running sum (from `carry`) exceeds target, or -1;
// *base gets the running sum before it.  If rounding hides the crossing inside
// the lane that holds it, that lane's last tile with a positive sum is taken.
__device__ __forceinline__ int walk_tile_block(const TileBlock& tb, int s0, double carry, double target, double* base)
{
    const int lane = threadIdx.x & 31;
    const unsigned hm = __ballot_sync(0xffffffffu, carry + tb.incl > target);
    if (!hm) return -1;
    const int l = __ffs(hm) - 1;
    int found = -1, lastpos = -1;
    double at = 0.0, lastat = 0.0;
    if (lane == l) {
        double run = carry + (tb.incl - tb.ls);
#pragma unroll
        for (int q = 0; q < kDrawQ; ++q) {
            if (found < 0 && tb.v[q] > 0.f) {
                if (run + (double)tb.v[q] > target) {
                    found = q;
                    at = run;
                } else {
                    lastpos = q;
                    lastat = run;
                }
            }
            run += (double)tb.v[q];
        }
        if (found < 0) {
            found = lastpos;
            at = lastat;
        }
    }
    found = __shfl_sync(0xffffffffu, found, l);
    *base = __shfl_sync(0xffffffffu, at, l);
    return found < 0 ? -1 : s0 + l * kDrawQ + found;
}

// Sum of all tile sums of a sequence, in the block order walk_tile_block uses.
__device__ double tiles_total(const float* w, int n, bool smem)
{
    double carry = 0.0;
    for (int s0 = 0; s0 < n; s0 += 32 * kDrawQ) {
        TileBlock tb;
        load_tile_block(tb, w, n, s0, smem);
        carry += __shfl_sync(0xffffffffu, tb.incl, 31);
    }
    return carry;
}

// The token inside tile ts: the first element whose running weight sum (from
// base) exceeds target, else the tile's last element with a positive weight.
template <int ESZ>
__device__ long long search_tile(const PassArgs& g, const SeqRec& rec, bool p_only, const uint4* tv,
                                 const uint4* dv, int ts, double base, double target)
{
    constexpr int VEC = 16 / ESZ;
    const int lane = threadIdx.x & 31;
    const long long q = (long long)ts * kTileVecs + lane;
    float w[VEC];
    double ls = 0.0;
    if (q < g.nq) {
        float xt[VEC], xd[VEC];
        unpack<ESZ>(__ldg(tv + q), xt);
        unpack<ESZ>(p_only ? make_uint4(0u, 0u, 0u, 0u) : __ldg(dv + q), xd);
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            w[e] = weight_of(rec, p_only, xt[e], p_only ? 0.f : xd[e]);
            ls += (double)w[e];
        }
    } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) w[e] = 0.f;
    }
    const double incl = warp_inclusive_scan(ls);
    double c = base + (incl - ls);
    int hit = -1, lastpos = -1;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        c += (double)w[e];
        if (hit < 0 && w[e] > 0.f && c > target) hit = e;
        if (w[e] > 0.f) lastpos = e;
    }
    const unsigned hm = __ballot_sync(0xffffffffu, hit >= 0);
    const unsigned lm = __ballot_sync(0xffffffffu, lastpos >= 0);
    if (hm) {
        const int l = __ffs(hm) - 1;
        return ((long long)ts * kTileVecs + l) * VEC + __shfl_sync(0xffffffffu, hit, l);
    }
    if (lm) {
        const int l = 31 - __clz(lm);
        return ((long long)ts * kTileVecs + l) * VEC + __shfl_sync(0xffffffffu, lastpos, l);
    }
    return -1;
}

// Weight sums of tiles [k0, k1) of the row pair into dst[k - k0], one per
// warp-tile: warp w takes tiles k0 + w, k0 + w + 8, ...; lane l vector 32k + l,
// U tiles per batch (the CTA's 16 warps per SM keep the loads in flight; an L1
// prefetch of the next batch measured no faster).  Loads allocate in L1, so the
// draw's second look at its tile often hits.  Vectors past the row read as -inf
// target logits (weight 0).
template <int ESZ, bool PONLY, int U>
__device__ __forceinline__ void tile_sums(const PassArgs& g, const SeqRec& rec, const uint4* tv, const uint4* dv,
                                          float* dst, int k0, int k1)
{
    constexpr int VEC = 16 / ESZ;
    constexpr int STEP = U * kWarps;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int kb = k0 + warp; kb < k1; kb += STEP) {
        uint4 vt[U], vd[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int k = kb + u * kWarps;
            const long long q = (long long)k * kTileVecs + lane;
            const bool ok = k < k1 && q < g.nq;
            vt[u] = ok ? __ldg(tv + q) : neg_inf_vec<ESZ>();
            if (!PONLY) vd[u] = ok ? __ldg(dv + q) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float xt[VEC], xd[VEC];
            float w[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            unpack<ESZ>(vt[u], xt);
            if (!PONLY) unpack<ESZ>(vd[u], xd);
#pragma unroll
            for (int e = 0; e < VEC; ++e) w[e] = weight_of(rec, PONLY, xt[e], PONLY ? 0.f : xd[e]);
            float s = tree8(w);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            const int k = kb + u * kWarps;
            if (lane == 0 && k < k1) dst[k - k0] = s;
        }
    }
}

// The vanished-residual fallback's tile sums of p_n (rare: kept out of line, so
// the registers the draw keeps live are saved around it instead of squeezing the
// main tile loop).
template <int ESZ>
__device__ __noinline__ void tile_sums_p(const PassArgs& g, const SeqRec rec, const uint4* tv, float* dst, int k0,
                                         int k1)
{
    tile_sums<ESZ, true, kTileU>(g, rec, tv, tv, dst, k0, k1);
}

// Per-sequence inputs and what follows from them alone, fetched and computed
// before sv_draw waits for sv_stream.  Lane j < gamma of every warp holds
// position j.
struct SeqPre {
    float T, khi, klo, ur;
    double rT;  // 1 / T
    double lu;  // log u_accept[b][j]
    int tok;    // draft token x_j
    int st;     // status bits the inputs alone decide
};

__device__ __forceinline__ SeqPre seq_pre(const TailArgs& a, int b)
{
    const int lane = threadIdx.x & 31;
    SeqPre s;
    s.T = __ldg(a.temperature + b);
    s.ur = __ldg(a.u_resample + b);
    s.tok = -1;
    float ua = 0.5f;
    if (lane < a.gamma) {
        s.tok = __ldg(a.tokens + (size_t)b * a.gamma + lane);
        ua = __ldg(a.u_accept + (size_t)b * a.gamma + lane);
    }
    const bool greedy = (s.T == 0.f);
    const bool tval = temperature_ok(s.T);
    s.khi = 0.f;
    s.klo = 0.f;
    s.rT = 0.0;
    if (tval && !greedy) {
        split_k(s.T, &s.khi, &s.klo);
        s.rT = 1.0 / (double)s.T;
    }
    s.lu = log((double)ua);
    int st = 0;
    if (!tval) {
        st = SV_ROW_BAD_TEMPERATURE;
    } else {
        if (__any_sync(0xffffffffu, lane < a.gamma && (s.tok < 0 || s.tok >= a.V))) st |= SV_ROW_BAD_TOKEN;
        // the uniforms stand for draws of U[0, 1): anything else (NaN included) is
        // an invalid input; a greedy sequence reads none
        if (!greedy && __any_sync(0xffffffffu, (lane < a.gamma && !(ua >= 0.f && ua < 1.f)) ||
                                                   !(s.ur >= 0.f && s.ur < 1.f)))
            st |= SV_ROW_BAD_UNIFORM;
    }
    s.st = st;
    return s;
}

// Per-row results of the finish, in each CTA's shared memory.
struct FinishSmem {
    double a2[kMaxRows];   // log2-normaliser of each row (NaN if bad)
    double sum[kMaxRows];  // sum relative to the integer offset
    float mk[kMaxRows];
    int arg[kMaxRows];
    int bad[kMaxRows];
    float gath[2 * SV_MAX_GAMMA];
    SeqRec rec;
    int st;
};

// Finish sequence b in one CTA (every CTA of the cluster does it, so none waits
// for another): warp w folds rows w, w + 8, ... (lane l reads slot l of each,
// every load in flight at once) in fp64; warp 0 forms every row's
// log2-normaliser (one row per lane), runs the log-space test at every draft
// position [FlashSpec, Metodologia 1, "Mecanismo"] with the gathered logits, and
// takes the first rejection from one ballot.  fs.rec and fs.st hold the outcome
// afterwards.  With `out`, also writes the accepted prefix, -1 padding,
// n_accepted and the normalisers (the status waits for the draw).
template <int ESZ>
__device__ __forceinline__ void finish_seq(const PassArgs& g, int b, const SeqPre& in, FinishSmem& fs, bool out)
{
    constexpr int kRowIter = (kMaxRows + kWarps - 1) / kWarps;
    const TailArgs& a = g.t;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gamma = a.gamma, R = a.R;
    const bool greedy = (in.T == 0.f);
    const bool tval = temperature_ok(in.T);
    const int rows_used = !tval ? 0 : (greedy ? gamma + 1 : R);

    const float4* pp = reinterpret_cast<const float4*>(g.part) + (size_t)b * R * kStreamSlots;
    const float4 kEmpty = make_float4(-INFINITY, 0.f, 0.f, __int_as_float(0x7fffffff));
    float4 q[kRowIter];
#pragma unroll
    for (int k = 0; k < kRowIter; ++k) {
        const int r = warp + kWarps * k;
        q[k] = r < rows_used ? __ldcg(pp + (size_t)r * kStreamSlots + lane) : kEmpty;
    }
    if (tid < 2 * gamma && tval && !greedy) fs.gath[tid] = __ldcg(g.gath + (size_t)b * 2 * gamma + tid);
#pragma unroll
    for (int k = 0; k < kRowIter; ++k) {
        const int r = warp + kWarps * k;
        if (r >= rows_used) break;
        if (greedy) {
            Amax A{q[k].x, __float_as_int(q[k].w), q[k].z != 0.f};
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ob = __shfl_xor_sync(0xffffffffu, A.best, o);
                const int oi = __shfl_xor_sync(0xffffffffu, A.idx, o);
                const int on = __shfl_xor_sync(0xffffffffu, A.nan, o);
                amax_merge(A, ob, oi, on);
            }
            if (lane == 0) {
                fs.arg[r] = A.idx;
                fs.bad[r] = A.nan || A.best == INFINITY || A.best == -INFINITY;
            }
        } else {
            const bool has = (q[k].x != -INFINITY);
            float MK = has ? q[k].y : -INFINITY;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) MK = fmaxf(MK, __shfl_xor_sync(0xffffffffu, MK, o));
            double S = has ? (double)q[k].z * pow2d(q[k].y - MK) : 0.0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
            if (lane == 0) {
                const bool bad = (MK == -INFINITY) || !isfinite(S) || !(S > 0.0);
                fs.bad[r] = bad;
                fs.mk[r] = MK;
                fs.sum[r] = S;
                fs.a2[r] = bad ? (double)NAN : (double)MK + log2(S);
            }
        }
    }
    __syncthreads();

    if (warp == 0) {
        int st = in.st;
        if (tval) {
            int badrow = 0;
            for (int r = lane; r < rows_used; r += 32) badrow |= fs.bad[r];
            if (__any_sync(0xffffffffu, badrow)) st |= SV_ROW_BAD_LOGITS;
        }
        bool acc = false;
        if (st == 0 && lane < gamma) {
            if (greedy) {
                acc = (in.tok == fs.arg[lane]);
            } else {
                const double lp = (double)fs.gath[lane] * in.rT - fs.a2[lane] * kLn2;
                const double lq = (double)fs.gath[gamma + lane] * in.rT - fs.a2[gamma + 1 + lane] * kLn2;
                acc = in.lu < (lp - lq);
            }
        }
        const unsigned mask = (gamma == 32) ? 0xffffffffu : ((1u << gamma) - 1u);
        const unsigned rej = __ballot_sync(0xffffffffu, !acc) & mask;
        const int n = (st != 0) ? 0 : (rej ? __ffs(rej) - 1 : gamma);
        if (lane == 0) {
            SeqRec rec;
            rec.mode = (st != 0 || greedy) ? kModeNone : (n < gamma ? kModeResidual : kModeBonus);
            rec.n = n;
            rec.k_hi = in.khi;
            rec.k_lo = in.klo;
            rec.mk_t = 0.f;
            rec.inv_s_t = 0.f;
            rec.mk_d = 0.f;
            rec.inv_s_d = 0.f;
            if (rec.mode != kModeNone) {
                rec.mk_t = fs.mk[n];
                rec.inv_s_t = (float)(1.0 / fs.sum[n]);
                if (rec.mode == kModeResidual) {
                    rec.mk_d = fs.mk[gamma + 1 + n];
                    rec.inv_s_d = (float)(1.0 / fs.sum[gamma + 1 + n]);
                }
            }
            fs.rec = rec;
            fs.st = st;
        }
        if (out) {
            // lane j < gamma holds draft token j; entry gamma is never a draft
            int32_t* ot = a.out_tokens + (size_t)b * (gamma + 1);
            for (int j = lane; j <= gamma; j += 32) {
                int v = -1;
                if (st == 0) {
                    if (j < n) v = in.tok;
                    else if (j == n && greedy) v = fs.arg[n];
                }
                ot[j] = v;  // a sampled extra token is written by the draw
            }
            if (lane == 0) a.out_n[b] = n;
        }
    }
    __syncthreads();
    if (out && a.out_log_norm) {
        double* ln = a.out_log_norm + (size_t)b * R;
        for (int r = tid; r < R; r += kPassThreads)
            ln[r] = (tval && !greedy && r < rows_used && !fs.bad[r]) ? fs.a2[r] * kLn2 : (double)NAN;
    }
}

// This CTA's tile sums in w[0, nt): their total (the order the walk uses); warp 0
// keeps the first block in tb0.
__device__ __forceinline__ double cta_tiles_total(TileBlock& tb0, const float* w, int nt, bool smem)
{
    load_tile_block(tb0, w, nt, 0, smem);
    return nt <= 32 * kDrawQ ? __shfl_sync(0xffffffffu, tb0.incl, 31) : tiles_total(w, nt, smem);
}

// The token of the CTA whose tile range holds u * S: walk its tile sums from
// `base` (the totals of the ranks before it), then the tile (warp 0 only).
template <int ESZ>
__device__ long long draw_in_cta(const PassArgs& g, const SeqRec& rec, bool p_only, const uint4* tv,
                                 const uint4* dv, const TileBlock& tb0, const float* w, int nt, bool smem, int k0,
                                 double base, double target)
{
    double at = 0.0;
    int ts = walk_tile_block(tb0, 0, base, target, &at);
    double carry = base + __shfl_sync(0xffffffffu, tb0.incl, 31);
    for (int s0 = 32 * kDrawQ; s0 < nt && ts < 0; s0 += 32 * kDrawQ) {
        TileBlock tb;
        load_tile_block(tb, w, nt, s0, smem);
        ts = walk_tile_block(tb, s0, carry, target, &at);
        carry += __shfl_sync(0xffffffffu, tb.incl, 31);
    }
    if (ts < 0) {
        // rounding put u * S past this CTA's last crossing: its last tile with a
        // positive sum, and in it the last token with a positive weight
        const int lane = threadIdx.x & 31;
        int last = -1;
        for (int kb = nt - 1; kb >= 0 && last < 0; kb -= 32) {
            const int k = kb - lane;
            const float v = k >= 0 ? (smem ? w[k] : __ldcg(w + k)) : 0.f;
            const unsigned m = __ballot_sync(0xffffffffu, v > 0.f);
            if (m) last = kb - (__ffs(m) - 1);
        }
        if (last < 0) return -1;
        return search_tile<ESZ>(g, rec, p_only, tv, dv, k0 + last, 0.0, (double)INFINITY);
    }
    return search_tile<ESZ>(g, rec, p_only, tv, dv, k0 + ts, at, target);
}

template <int ESZ>
__global__ void __launch_bounds__(kPassThreads, 2) sv_draw(const __grid_constant__ PassArgs g)
{
    __shared__ FinishSmem s_fin;
    __shared__ float s_tiles[kTileSmem];         // this CTA's tile sums
    __shared__ double s_tot[3][kMaxCluster];     // every rank's total: two alternating, one for the fallback
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank(), cs = (int)cluster.num_blocks();
    const int cid = blockIdx.x / cs, nclusters = gridDim.x / cs;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TailArgs& t = g.t;
    const int per = (g.NT2 + cs - 1) / cs;
    const int k0 = min(g.NT2, rank * per), k1 = min(g.NT2, k0 + per), nt = k1 - k0;
    const bool smem = per <= kTileSmem;

    // the first sequence's inputs are not sv_stream's outputs: fetch them and work
    // out what they decide before waiting for sv_stream's writes to be visible
    SeqPre in = seq_pre(t, min(cid, g.B - 1));
    cluster.sync();  // every CTA of the cluster runs before any writes another's shared memory
    asm volatile("griddepcontrol.wait;" ::: "memory");

    int par = 0;
    for (int b = cid; b < g.B; b += nclusters, par ^= 1) {
        if (b != cid) {
            __syncthreads();  // warp 0 is done with the previous sequence's shared memory
            in = seq_pre(t, b);
        }
        finish_seq<ESZ>(g, b, in, s_fin, rank == 0);
        const SeqRec rec = s_fin.rec;
        const bool bonus = (rec.mode == kModeBonus);
        const uint4* tv = reinterpret_cast<const uint4*>(row_ptr<ESZ>(t, b, rec.n));
        const uint4* dv = bonus ? tv : reinterpret_cast<const uint4*>(row_ptr<ESZ>(t, b, t.gamma + 1 + rec.n));
        float* w = smem ? s_tiles : g.tsum + (size_t)b * g.NT2 + k0;
        if (rec.mode == kModeResidual) tile_sums<ESZ, false, kTileU>(g, rec, tv, dv, w, k0, k1);
        else if (rec.mode == kModeBonus) tile_sums<ESZ, true, kTileU>(g, rec, tv, tv, w, k0, k1);
        __syncthreads();
        TileBlock tb0;
        if (warp == 0) {
            const double tot = rec.mode != kModeNone ? cta_tiles_total(tb0, w, nt, smem) : 0.0;
            if (lane < cs) *cluster.map_shared_rank(&s_tot[par][rank], lane) = tot;
        }
        cluster.sync();  // every rank's total is in every rank's s_tot[par]
        bool p_only = bonus;
        int flag = 0;
        int slot = par;
        if (rec.mode != kModeNone) {
            double S = 0.0;
            for (int r = 0; r < cs; ++r) S += s_tot[slot][r];
            if (!bonus && !(S >= kResidualMin)) {
                // the residual vanished (below kResidualMin): draw from p_n instead
                flag = SV_ROW_RESIDUAL_ZERO;
                p_only = true;
                tile_sums_p<ESZ>(g, rec, tv, w, k0, k1);
                __syncthreads();
                if (warp == 0) {
                    const double tot = cta_tiles_total(tb0, w, nt, smem);
                    if (lane < cs) *cluster.map_shared_rank(&s_tot[2][rank], lane) = tot;
                }
                cluster.sync();
                slot = 2;
                S = 0.0;
                for (int r = 0; r < cs; ++r) S += s_tot[slot][r];
            }
            // the rank whose range holds u * S (in the sum's own order); if rounding
            // leaves none, the last rank with a positive total
            const double target = (double)in.ur * S;
            double pre = 0.0, base = 0.0;
            int rs = -1, rl = -1;
            double basel = 0.0;
            for (int r = 0; r < cs; ++r) {
                const double v = s_tot[slot][r];
                if (rs < 0 && pre + v > target) {
                    rs = r;
                    base = pre;
                }
                if (v > 0.0) {
                    rl = r;
                    basel = pre;
                }
                pre += v;
            }
            if (rs < 0) {
                rs = rl;
                base = basel;
            }
            if (rank == rs && warp == 0) {
                const long long token = draw_in_cta<ESZ>(g, rec, p_only, tv, p_only ? tv : dv, tb0, w, nt, smem, k0,
                                                         base, target);
                if (lane == 0) t.out_tokens[(size_t)b * (t.gamma + 1) + rec.n] = (int)token;
            }
        }
        if (rank == 0 && threadIdx.x == 0 && t.out_status) t.out_status[b] = s_fin.st | flag;
    }
}

}  // namespace sv
