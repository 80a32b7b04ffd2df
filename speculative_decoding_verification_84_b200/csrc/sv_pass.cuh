// sv_pass.cuh -- the streaming path for rows that are 16-byte aligned and at
// least 4 KB: two persistent kernels.
//
//   sv_pass1  the rows, in sequence order, form one stream of 16-byte vectors;
//             warp w of the grid takes the contiguous span [w*S, (w+1)*S) and
//             walks it on its own -- no barrier, no atomic -- 8 vectors per lane
//             per batch, keeping per-lane online log-sum-exp state of l/T (the
//             exponent arguments and sums on packed fp32 pairs) or the first
//             argmax (T_b = 0).  Where its span crosses a row boundary (at most a
//             few times) the warp reduces with shuffles and writes one Partial for
//             that row segment.  A barrier per chunk would make every CTA wait for
//             its slowest load; independent warps keep HBM busy.
//             The warp whose segment holds a row's draft token x_j also stores
//             the logit l[x_j] for the accept test.
//   sv_pass2  one thread-block cluster per sequence b (clusters loop over the
//             sequences): rank 0 finishes b -- fp64 combine of its partials,
//             log-space accept scan [FlashSpec, Metodologia 1] (sequence_tail) --
//             and a cluster barrier (hardware, no polling) hands the outcome to
//             the cluster through distributed shared memory.  The cluster's CTAs
//             then split the row pair the extra token is drawn from (residual
//             max(0, p_n - q_n), or p_gamma for the bonus) [Speculative
//             Speculative Decoding, Metodologia 2], each warp turning 32
//             consecutive vectors (a tile) into one fp32 weight sum; after a
//             second cluster barrier rank 0 draws the token by inverse CDF over
//             b's tile sums.
// Pass 1's grid holds as many CTAs as are resident at once (4 per SM at 256
// threads and at most 64 registers), so every warp streams from start to end.
// Pass 2 runs 2 CTAs per SM (the finish and the draw run in registers), in
// clusters of up to 8 sized so that one wave covers the batch when it can; it is
// launched as a programmatic dependent of pass 1: its CTAs start as pass-1 CTAs
// leave and wait (griddepcontrol.wait) for all of pass 1 before reading.
#pragma once

#include "sv_common.cuh"
#include "sv_generic.cuh"

#include <cooperative_groups.h>

namespace sv {

namespace cg = cooperative_groups;

constexpr int kPassThreads = 256;                  // = kThreads: reduce_lse / reduce_amax apply
constexpr int kP1Vec = 8;                          // 16-byte vectors per lane per pass-1 batch
constexpr int kMaxCluster = 8;                     // pass-2 cluster size limit (portable)
constexpr int kTileSmem = 4096;                    // tile sums kept in rank 0's shared memory up to this many
constexpr int kTileVecs = 32;                      // vectors per tile (one per lane)
constexpr int kStreamMinRowBytes = 4096;           // shorter rows take the generic path
constexpr int kDrawQ = 16;                         // tile sums per lane per draw block
constexpr int kSpanMin = 512;                      // shortest pass-1 span (vectors): bounds slots per row

static_assert(kPassThreads == kThreads, "block reductions assume kThreads threads");

struct PassArgs {
    TailArgs t;              // t.nc = partial slots per row (stride and count); t.gath = gath
    Partial* part;           // [B][R][t.nc]; the slots no span fills hold empty partials
    float* gath;             // [B][2*gamma] the accept test's logits, written by pass 1
    float* tsum;             // [B][NT2] weight sum of each tile
    const float* u_resample;
    long long nq;            // 16-byte vectors per row
    long long S;             // vectors per warp span (pass 1)
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

// ----------------------------------------------------------------------------- pass 1

// One row segment [q0, q0 + n) of row (b, r) by one warp: batches of 32*kP1Vec
// vectors (vector q0 + j*256 + u*32 + lane), reduced with shuffles; lane 0
// writes the Partial.
template <int ESZ>
__device__ __forceinline__ void pass1_segment(const PassArgs& g, int b, int r, long long q0, int n, Partial* dst)
{
    constexpr int VEC = 16 / ESZ;
    constexpr int kStep = 32 * kP1Vec;
    const TailArgs& a = g.t;
    const int lane = threadIdx.x & 31;
    const float T = __ldg(a.temperature + b);
    const bool greedy = (T == 0.f);
    if (!temperature_ok(T) || (greedy && r > a.gamma)) return;  // a row the finish will not read
    const uint4* p = reinterpret_cast<const uint4*>(row_ptr<ESZ>(a, b, r)) + q0;
    if (greedy) {
        Amax A{-INFINITY, 0x7fffffff, 0};
        const int e0 = (int)(q0 * VEC);
        for (int j0 = 0; j0 < n; j0 += kStep) {
            uint4 v[kP1Vec];
#pragma unroll
            for (int u = 0; u < kP1Vec; ++u) {
                const int i = j0 + u * 32 + lane;
                v[u] = i < n ? ld_stream(p + i) : neg_inf_vec<ESZ>();
            }
#pragma unroll
            for (int u = 0; u < kP1Vec; ++u) {
                float x[VEC];
                unpack<ESZ>(v[u], x);
                const int i0 = e0 + (j0 + u * 32 + lane) * VEC;
                // fill elements (-inf past the segment) have larger indices than
                // the real ones, so they never win a tie
#pragma unroll
                for (int e = 0; e < VEC; ++e) amax_add(A, x[e], i0 + e);
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
    } else {
        float khi, klo;
        split_k(T, &khi, &klo);
        Lse L;
        lse_init(L);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j0 = 0; j0 < n; j0 += kStep) {
            uint4 v[kP1Vec];
            if (j0 + kStep <= n) {
#pragma unroll
                for (int u = 0; u < kP1Vec; ++u) v[u] = ld_stream(p + j0 + u * 32 + lane);
            } else {
#pragma unroll
                for (int u = 0; u < kP1Vec; ++u) {
                    const int i = j0 + u * 32 + lane;
                    v[u] = i < n ? ld_stream(p + i) : neg_inf_vec<ESZ>();  // -inf: weight 0
                }
            }
            lse_group2<ESZ, kP1Vec>(L, acc, v, khi, klo);
        }
        lse_fold(L, acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float om = __shfl_xor_sync(0xffffffffu, L.m, o);
            const float omk = __shfl_xor_sync(0xffffffffu, L.mk, o);
            const float os = __shfl_xor_sync(0xffffffffu, L.s, o);
            lse_merge(L, om, omk, os);
        }
        if (lane == 0) {
            *dst = Partial{L.m, L.mk, L.m == -INFINITY ? 0.f : L.s, 0};
            // the accept test's logit l[x_j] of this row, if the segment holds it
            // (target rows j < gamma and draft rows j; the bonus row has no token)
            if (r != a.gamma) {
                const int j = r < a.gamma ? r : r - a.gamma - 1;
                const int x = __ldg(a.tokens + (size_t)b * a.gamma + j);
                const long long e = (long long)x - q0 * VEC;
                if (x >= 0 && x < a.V && e >= 0 && e < (long long)n * VEC)
                    g.gath[(size_t)b * 2 * a.gamma + (r < a.gamma ? j : a.gamma + j)] =
                        load_logit<ESZ>(p, (size_t)e);
            }
        }
    }
}

template <int ESZ>
__global__ void __launch_bounds__(kPassThreads, 4) sv_pass1(PassArgs g)
{
    const TailArgs& a = g.t;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // pass 2 may be scheduled
    const long long w = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const long long NQ = (long long)g.B * a.R * g.nq;
    long long v0 = w * g.S;
    const long long v1 = min(v0 + g.S, NQ);
    while (v0 < v1) {
        const long long row = v0 / g.nq;  // global row index b*R + r
        const long long end = min(v1, (row + 1) * g.nq);
        const int b = (int)(row / a.R), r = (int)(row - (long long)b * a.R);
        // spans s0 .. w meet the row so far: this segment is its slot w - s0
        const int slot = (int)(w - (row * g.nq) / g.S);
        Partial* prow = g.part + (size_t)row * a.nc;
        pass1_segment<ESZ>(g, b, r, v0 - row * g.nq, (int)(end - v0), prow + slot);
        // the span that ends the row marks the row's remaining slots empty, so the
        // finish reads a fixed t.nc slots per row
        const int lane = threadIdx.x & 31;
        if (end == (row + 1) * g.nq)
            for (int k = slot + 1 + lane; k < a.nc; k += 32) prow[k] = Partial{-INFINITY, 0.f, 0.f, 0x7fffffff};
        v0 = end;
    }
}

// ----------------------------------------------------------------------------- pass 2 and the draw

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
    double s = 0.0;
#pragma unroll
    for (int q = 0; q < kDrawQ; ++q) s += (double)tb.v[q];
    tb.ls = s;
    tb.incl = warp_inclusive_scan(s);
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
__device__ __noinline__ void pass2_draw(const PassArgs& g, int b, const SeqRec& rec, float* ws, bool smem)
{
    __shared__ double s_S;
    const TailArgs& t = g.t;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = g.NT2;
    const bool bonus = (rec.mode == kModeBonus);
    const uint4* tv = reinterpret_cast<const uint4*>(row_ptr<ESZ>(t, b, rec.n));
    const uint4* dv = bonus ? tv : reinterpret_cast<const uint4*>(row_ptr<ESZ>(t, b, t.gamma + 1 + rec.n));
    if (warp == 0) {
        const double S = tiles_total(ws, n, smem);
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
    }
    if (warp != 0) return;
    const double S = flag ? tiles_total(ws, n, smem) : s_S;
    const double target = (double)__ldg(g.u_resample + b) * S;
    int ts = -1;
    double base = 0.0, carry = 0.0;
    for (int s0 = 0; s0 < n && ts < 0; s0 += 32 * kDrawQ) {
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
// tiles k0 + 8*(4j + u) + w (u < 4), lane l vector 32k + l, so each lane has 4
// (or 8, with the draft row) loads in flight.  Vectors past the row read as -inf
// target logits, whose weight is 0.
template <int ESZ, bool PONLY>
__device__ void tile_range(const PassArgs& g, const SeqRec& rec, const uint4* tv, const uint4* dv, float* dst,
                           int k0, int k1)
{
    constexpr int VEC = 16 / ESZ;
    constexpr int U = 4;
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

template <int ESZ>
__device__ __noinline__ void pass2_finish(const PassArgs& g, int b, TailSmem& ts, SeqRec* rec_out)
{
    const TailArgs& a = g.t;
    sequence_tail<ESZ, kPassThreads, BlockSync>(a, b, threadIdx.x, FloatPartials{a.part}, ts);
    __syncthreads();
    if (threadIdx.x == 0) *rec_out = ts.rec;
}

template <int ESZ>
__global__ void __launch_bounds__(kPassThreads, 2) sv_pass2(PassArgs g)
{
    __shared__ TailSmem s_tail;
    __shared__ SeqRec s_rec;
    __shared__ float s_tiles[kTileSmem];  // rank 0: b's tile sums, written by the whole cluster
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank(), cs = (int)cluster.num_blocks();
    const int cid = blockIdx.x / cs, nclusters = gridDim.x / cs;
    const TailArgs& t = g.t;
    const bool tiles_in_smem = g.NT2 <= kTileSmem;
    float* tiles0 = cluster.map_shared_rank(s_tiles, 0);  // rank 0's buffer, from any rank

    // wait until pass 1 has completed and its writes are visible (a no-op when
    // this launch did not overlap pass 1)
    asm volatile("griddepcontrol.wait;" ::: "memory");

    for (int b = cid; b < g.B; b += nclusters) {
        if (rank == 0) pass2_finish<ESZ>(g, b, s_tail, &s_rec);
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
            if (bonus) tile_range<ESZ, true>(g, rec, tv, tv, dst, k0, k1);
            else tile_range<ESZ, false>(g, rec, tv, dv, dst, k0, k1);
        }
        cluster.sync();  // every tile sum of b is visible to rank 0
        if (rank == 0 && rec.mode != kModeNone) pass2_draw<ESZ>(g, b, rec, tiles_in_smem ? s_tiles : dst, tiles_in_smem);
        // rank 0's s_rec and s_tiles are rewritten for the next sequence only
        // after the next iteration's finish, which the other ranks wait for
    }
}

}  // namespace sv
