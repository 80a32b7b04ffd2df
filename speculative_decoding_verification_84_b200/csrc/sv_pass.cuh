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
//              sequences): rank 0 finishes b -- fp64 combine of the partials
//              (every load of the finish in flight at once), the log-space
//              accept test [FlashSpec, Metodologia 1] with the first rejection
//              from one ballot -- and a cluster barrier hands the outcome to the
//              cluster through distributed shared memory; the cluster's CTAs then
//              split the draw rows (residual max(0, p_n - q_n), or p_gamma for
//              the bonus token) [Speculative Speculative Decoding, Metodologia 2,
//              "Conceito Central"; Desafios 2, "Amostragem Saguaro"] into tiles
//              of 32 vectors, one fp32 weight sum per tile into rank 0's shared
//              memory; after a second barrier rank 0 draws the token by inverse
//              CDF over the tile sums.
// sv_stream triggers its dependents at entry, so sv_draw's CTAs start as
// sv_stream's leave; they fetch their sequence's inputs and then wait
// (griddepcontrol.wait) for all of sv_stream before reading its partials.
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
constexpr int kTileSmem = 4096;                    // tile sums kept in rank 0's shared memory up to this many
constexpr int kTileVecs = 32;                      // vectors per tile (one per lane)
constexpr int kTileBatch = 8;                      // tiles per warp in flight in sv_draw
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
#pragma unroll
            for (int u = 0; u < kStreamVec; ++u) {
                float xv[VEC];
                unpack<ESZ>(v[u], xv);
                const int i0 = e0 + (j0 + u * 32 + lane) * VEC;
                // fill elements (-inf past the segment) have larger indices than
                // the real ones, so they never win a tie
#pragma unroll
                for (int e = 0; e < VEC; ++e) amax_add(A, xv[e], i0 + e);
            }
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
        unpack<ESZ>(ld_stream(tv + q), xt);
        unpack<ESZ>(p_only ? make_uint4(0u, 0u, 0u, 0u) : ld_stream(dv + q), xd);
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

// Weight sums of tiles k = first, first + stride, ... (< NT2) of the row pair,
// one warp per tile: lane l takes vector 32k + l; vectors past the row read as
// -inf target logits, whose weight is 0.
template <int ESZ>
__device__ void tile_sums_strided(const PassArgs& g, const SeqRec& rec, bool p_only, const uint4* tv,
                                  const uint4* dv, float* dst, int first, int stride)
{
    constexpr int VEC = 16 / ESZ;
    const int lane = threadIdx.x & 31;
    for (int k = first; k < g.NT2; k += stride) {
        const long long q = (long long)k * kTileVecs + lane;
        const bool ok = q < g.nq;
        float xt[VEC], xd[VEC];
        float w[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        unpack<ESZ>(ok ? ld_stream(tv + q) : neg_inf_vec<ESZ>(), xt);
        unpack<ESZ>((ok && !p_only) ? ld_stream(dv + q) : make_uint4(0u, 0u, 0u, 0u), xd);
#pragma unroll
        for (int e = 0; e < VEC; ++e) w[e] = weight_of(rec, p_only, xt[e], p_only ? 0.f : xd[e]);
        float s = tree8(w);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) dst[k] = s;
    }
}

// Inverse CDF for sequence b, run by the whole CTA (warp 0 does the search): the
// smallest token k with C_k > u * S over b's tile sums; a vanished residual
// (S = 0) falls back to p_n, whose tile sums the CTA computes first.
template <int ESZ>
__device__ __noinline__ void pass2_draw(const PassArgs& g, int b, const SeqRec& rec, float* ws, bool smem, float ur)
{
    __shared__ double s_S;
    const TailArgs& t = g.t;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = g.NT2;
    const bool bonus = (rec.mode == kModeBonus);
    const uint4* tv = reinterpret_cast<const uint4*>(row_ptr<ESZ>(t, b, rec.n));
    const uint4* dv = bonus ? tv : reinterpret_cast<const uint4*>(row_ptr<ESZ>(t, b, t.gamma + 1 + rec.n));
    // warp 0 keeps the first block of tile sums in registers for the walk
    TileBlock tb0;
    if (warp == 0) {
        load_tile_block(tb0, ws, n, 0, smem);
        const double S = n <= 32 * kDrawQ ? __shfl_sync(0xffffffffu, tb0.incl, 31) : tiles_total(ws, n, smem);
        if (lane == 0) s_S = S;
    }
    __syncthreads();
    bool p_only = bonus;
    int flag = 0;
    if (!(s_S >= kResidualMin) && !bonus) {
        // the residual vanished (below kResidualMin): draw from p_n instead
        flag = SV_ROW_RESIDUAL_ZERO;
        p_only = true;
        tile_sums_strided<ESZ>(g, rec, true, tv, tv, ws, warp, kWarps);
        __syncthreads();
        if (warp == 0) load_tile_block(tb0, ws, n, 0, smem);
    }
    if (warp != 0) return;
    const double S = flag ? tiles_total(ws, n, smem) : s_S;
    const double target = (double)__shfl_sync(0xffffffffu, ur, 0) * S;
    double base = 0.0;
    int ts = walk_tile_block(tb0, 0, 0.0, target, &base);
    double carry = __shfl_sync(0xffffffffu, tb0.incl, 31);
    for (int s0 = 32 * kDrawQ; s0 < n && ts < 0; s0 += 32 * kDrawQ) {
        TileBlock tb;
        load_tile_block(tb, ws, n, s0, smem);
        ts = walk_tile_block(tb, s0, carry, target, &base);
        carry += __shfl_sync(0xffffffffu, tb.incl, 31);
    }
    const long long token = ts >= 0 ? search_tile<ESZ>(g, rec, p_only, tv, dv, ts, base, target) : -1;
    if (lane == 0) {
        t.out_tokens[(size_t)b * (t.gamma + 1) + rec.n] = (int)token;
        if (flag && t.out_status) t.out_status[b] |= flag;
    }
}

// Weight sums of tiles [k0, k1) of the row pair, one per warp-tile: warp w takes
// tiles k0 + 8*(U*j + u) + w (u < U), lane l vector 32k + l, so each lane has U
// (or 2U, with the draft row) loads in flight.  Vectors past the row read as
// -inf target logits, whose weight is 0.
template <int ESZ, bool PONLY, int U>
__device__ void tile_range(const PassArgs& g, const SeqRec& rec, const uint4* tv, const uint4* dv, float* dst,
                           int k0, int k1)
{
    constexpr int VEC = 16 / ESZ;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int kb = k0 + warp; kb < k1; kb += U * kWarps) {
        uint4 vt[U], vd[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int k = kb + u * kWarps;
            const long long q = (long long)k * kTileVecs + lane;
            const bool ok = k < k1 && q < g.nq;
            vt[u] = ok ? ld_stream(tv + q) : neg_inf_vec<ESZ>();
            if (!PONLY) vd[u] = ok ? ld_stream(dv + q) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float xt[VEC], xd[VEC];
            float w[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            unpack<ESZ>(vt[u], xt);
            if (!PONLY) unpack<ESZ>(vd[u], xd);
#pragma unroll
            for (int e = 0; e < VEC; ++e) w[e] = weight_of(rec, PONLY, xt[e], PONLY ? 0.f : xd[e]);
            float sum = tree8(w);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            const int k = kb + u * kWarps;
            if (lane == 0 && k < k1) dst[k] = sum;
        }
    }
}


// What the finish of one sequence needs from the inputs, fetched before
// sv_draw waits for sv_stream (lane j < gamma of warp 0 holds position j).
struct SeqIn {
    float T;
    int tok;
    float ua;
    float ur;
};

__device__ __forceinline__ SeqIn load_seq_in(const TailArgs& a, int b)
{
    const int tid = threadIdx.x;
    SeqIn in;
    in.T = __ldg(a.temperature + b);
    in.tok = -1;
    in.ua = 0.5f;
    in.ur = 0.5f;
    if (tid < a.gamma) {
        in.tok = __ldg(a.tokens + (size_t)b * a.gamma + tid);
        in.ua = __ldg(a.u_accept + (size_t)b * a.gamma + tid);
    }
    if (tid == 0) in.ur = __ldg(a.u_resample + b);
    return in;
}

// Per-row results of the finish (shared memory of rank 0).
struct FinishSmem {
    double a2[kMaxRows];   // log2-normaliser of each row (NaN if bad)
    double sum[kMaxRows];  // sum relative to the integer offset
    float mk[kMaxRows];
    int arg[kMaxRows];
    int bad[kMaxRows];
    float gath[2 * SV_MAX_GAMMA];
    int status, n;
    float ur;  // u_resample of the sequence, for the draw
};

// Finish sequence b with one CTA: warp w folds rows w, w + 8, ... (lane l reads
// slot l of each, every load in flight at once) in fp64; gathers log p_j(x_j)
// and log q_j(x_j) [FlashSpec, Metodologia 1, "Mecanismo"]; warp 0 runs the
// log-space test at every draft position and takes the first rejection from one
// ballot; writes the accepted prefix, -1 padding, n_accepted, status and
// normalisers, and the draw record into *rec_out.
template <int ESZ>
__device__ __noinline__ void finish_cta(const PassArgs& g, int b, const SeqIn& in, FinishSmem& fs, SeqRec* rec_out)
{
    constexpr int kRowIter = (kMaxRows + kWarps - 1) / kWarps;
    const TailArgs& a = g.t;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gamma = a.gamma, R = a.R;
    const float T = in.T;
    const bool greedy = (T == 0.f);
    const bool tval = temperature_ok(T);
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
                fs.bad[r] = (MK == -INFINITY) || !isfinite(S) || !(S > 0.0);
                fs.mk[r] = MK;
                fs.sum[r] = S;
            }
        }
    }
    __syncthreads();

    if (warp == 0) {
        // every row's log2-normaliser at once, one row per lane
        if (!greedy)
            for (int r = lane; r < rows_used; r += 32)
                fs.a2[r] = fs.bad[r] ? (double)NAN : (double)fs.mk[r] + log2(fs.sum[r]);
        __syncwarp();
        int st = 0;
        const int x_j = (lane < gamma) ? in.tok : -1;
        if (!tval) {
            st = SV_ROW_BAD_TEMPERATURE;
        } else {
            const int badtok = (lane < gamma) && (x_j < 0 || x_j >= a.V);
            int badrow = 0;
            for (int r = lane; r < rows_used; r += 32) badrow |= fs.bad[r];
            // the uniforms stand for draws of U[0, 1): anything else (NaN included)
            // is an invalid input (a greedy sequence reads none)
            int bad_u = 0;
            if (!greedy) {
                if (lane < gamma) bad_u = !(in.ua >= 0.f && in.ua < 1.f);
                if (lane == 0) bad_u |= !(in.ur >= 0.f && in.ur < 1.f);
            }
            if (__any_sync(0xffffffffu, badtok)) st |= SV_ROW_BAD_TOKEN;
            if (__any_sync(0xffffffffu, badrow)) st |= SV_ROW_BAD_LOGITS;
            if (__any_sync(0xffffffffu, bad_u)) st |= SV_ROW_BAD_UNIFORM;
        }
        bool acc = false;
        if (st == 0 && lane < gamma) {
            if (greedy) {
                acc = (x_j == fs.arg[lane]);
            } else {
                const double rT = 1.0 / (double)T;
                const double lp = (double)fs.gath[lane] * rT - fs.a2[lane] * kLn2;
                const double lq = (double)fs.gath[gamma + lane] * rT - fs.a2[gamma + 1 + lane] * kLn2;
                acc = log((double)in.ua) < (lp - lq);
            }
        }
        const unsigned mask = (gamma == 32) ? 0xffffffffu : ((1u << gamma) - 1u);
        const unsigned rej = __ballot_sync(0xffffffffu, !acc) & mask;
        const int n = (st != 0) ? 0 : (rej ? __ffs(rej) - 1 : gamma);
        if (lane == 0) {
            fs.status = st;
            fs.n = n;
            fs.ur = in.ur;
        }
        // lane j < gamma holds draft token j (prefetched); entry gamma is never a draft
        int32_t* ot = a.out_tokens + (size_t)b * (gamma + 1);
        for (int j = lane; j <= gamma; j += 32) {
            int v = -1;
            if (st == 0) {
                if (j < n) v = x_j;
                else if (j == n && greedy) v = fs.arg[n];
            }
            ot[j] = v;  // a sampled extra token is written by the draw
        }
    }
    __syncthreads();

    const int st = fs.status, n = fs.n;
    if (a.out_log_norm) {
        double* ln = a.out_log_norm + (size_t)b * R;
        for (int r = tid; r < R; r += kPassThreads)
            ln[r] = (tval && !greedy && !fs.bad[r]) ? fs.a2[r] * kLn2 : (double)NAN;
    }
    if (tid == 0) {
        a.out_n[b] = n;
        if (a.out_status) a.out_status[b] = st;
        SeqRec rec;
        rec.mode = (st != 0 || greedy) ? kModeNone : (n < gamma ? kModeResidual : kModeBonus);
        rec.n = n;
        rec.mk_t = 0.f;
        rec.inv_s_t = 0.f;
        rec.mk_d = 0.f;
        rec.inv_s_d = 0.f;
        rec.k_hi = 0.f;
        rec.k_lo = 0.f;
        if (rec.mode != kModeNone) {
            split_k(T, &rec.k_hi, &rec.k_lo);
            rec.mk_t = fs.mk[n];
            rec.inv_s_t = (float)(1.0 / fs.sum[n]);
            if (rec.mode == kModeResidual) {
                rec.mk_d = fs.mk[gamma + 1 + n];
                rec.inv_s_d = (float)(1.0 / fs.sum[gamma + 1 + n]);
            }
        }
        *rec_out = rec;
    }
}

template <int ESZ>
__global__ void __launch_bounds__(kPassThreads, 2) sv_draw(const __grid_constant__ PassArgs g)
{
    __shared__ FinishSmem s_fin;
    __shared__ SeqRec s_rec;
    __shared__ float s_tiles[kTileSmem];  // rank 0: b's tile sums, written by the whole cluster
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank(), cs = (int)cluster.num_blocks();
    const int cid = blockIdx.x / cs, nclusters = gridDim.x / cs;
    const TailArgs& t = g.t;
    const bool tiles_in_smem = g.NT2 <= kTileSmem;
    float* tiles0 = cluster.map_shared_rank(s_tiles, 0);  // rank 0's buffer, from any rank

    // the first sequence's inputs are not sv_stream's outputs: fetch them before
    // waiting for sv_stream to complete and its writes to be visible
    SeqIn in = cid < g.B ? load_seq_in(t, cid) : SeqIn{0.f, -1, 0.5f, 0.5f};
    asm volatile("griddepcontrol.wait;" ::: "memory");

    for (int b = cid; b < g.B; b += nclusters) {
        if (b != cid) in = load_seq_in(t, b);
        if (rank == 0) finish_cta<ESZ>(g, b, in, s_fin, &s_rec);
        cluster.sync();  // rank 0's outcome is visible to the cluster
        const SeqRec rec = *cluster.map_shared_rank(&s_rec, 0);
        float* dst = tiles_in_smem ? tiles0 : g.tsum + (size_t)b * g.NT2;
        if (rec.mode != kModeNone) {
            const bool bonus = (rec.mode == kModeBonus);
            const uint4* tv = reinterpret_cast<const uint4*>(row_ptr<ESZ>(t, b, rec.n));
            const uint4* dv = bonus ? tv : reinterpret_cast<const uint4*>(row_ptr<ESZ>(t, b, t.gamma + 1 + rec.n));
            // this CTA's share of the tiles
            const int per = (g.NT2 + cs - 1) / cs;
            const int k0 = rank * per, k1 = min(g.NT2, k0 + per);
            if (bonus) tile_range<ESZ, true, kTileBatch>(g, rec, tv, tv, dst, k0, k1);
            else tile_range<ESZ, false, kTileBatch>(g, rec, tv, dv, dst, k0, k1);
        }
        cluster.sync();  // every tile sum of b is visible to rank 0
        if (rank == 0 && rec.mode != kModeNone)
            pass2_draw<ESZ>(g, b, rec, tiles_in_smem ? s_tiles : dst, tiles_in_smem, s_fin.ur);
        // rank 0's s_rec and s_tiles are rewritten for the next sequence only
        // after the next iteration's finish, which the other ranks wait for
    }
}

}  // namespace sv
