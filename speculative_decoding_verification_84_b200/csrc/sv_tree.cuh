// sv_tree.cuh -- verification of a token tree, and pruning by path probability
// [SpecLA, Metodologia 1, "Kernels de Verificacao de Topologia Conscientes":
// drafts shaped as chains or as branching trees; Metodologia 3, "Poda Guiada por
// Confianca": paths of low cumulative draft log-probability are removed before
// verification; Speculative Speculative Decoding, "Significado e Impacto": the
// method is compatible with token trees].
//
// The rule (the multi-candidate form of the speculative-sampling test): at node
// c, P starts as the target's p at c; the children of c are tested in index
// order, child x accepted iff log u_x < log P(tok_x) - log q(tok_x); after a
// rejection P becomes norm(max(0, P - q)) (unchanged, status bit 8, when that
// mass is below 2^-18); an accepted child becomes c; when c has no child left
// the extra token is drawn from P by the inverse CDF with u_resample.  T = 0:
// the first child whose token is the first argmax of target row c.  A chain
// is exactly spec_verify's case.
//
//   sv_tree         one thread-block cluster of CL CTAs per sequence walks the
//                   tree.  The CTAs split the vocabulary (CTA r owns a contiguous
//                   range of 16-byte groups, warp w a contiguous part of it, lane
//                   l every 32nd group of that part), so every pass over a row
//                   is spread over CL SMs.  Per visited node: one pass over
//                   target row c (and draft row c if c has children) gives the
//                   log-normalisers; each rejection costs one more pass (the
//                   residual mass, from L2); the draw one more (per-CTA sums,
//                   then the CTA holding u*S walks its warps, blocks, lanes and
//                   elements).  Partial results cross the cluster through
//                   distributed shared memory: every CTA pushes its part into
//                   every CTA's buffer, one cluster barrier, and every CTA folds
//                   the parts in rank order -- so every CTA takes the same
//                   decisions and no further broadcast is needed.  Inside a CTA
//                   the scalar work (the folds, the tests) is done once, by warp
//                   0 or thread 0, and shared through shared memory.  Only the
//                   rows of the nodes the walk visits are read.
//   sv_tree_prune_rows / sv_tree_prune_walk
//                   the draft's log q_c(tok_i) for every node i with parent c
//                   (one CTA per (sequence, parent row)), then the cumulative
//                   sums and the keep mask along the parent order (one warp per
//                   sequence, in shared memory).
#pragma once

#include <cooperative_groups.h>

#include "sv_common.cuh"

namespace sv {

namespace cgt = cooperative_groups;

constexpr int kTreeThreads = 512;
constexpr int kTreeWarps = kTreeThreads / 32;
constexpr int kTreeMaxNodes = 64;
constexpr int kTreeMaxCluster = 8;
constexpr int kTreeBatch = 2;  // groups per lane loaded before any is used
constexpr int kPruneThreads = 256;

struct TreeArgs {
    const void* tgt;
    const void* dft;
    const int32_t* parent;
    const int32_t* tokens;
    const int32_t* keep;  // optional
    const float* temperature;
    const float* u_accept;
    const float* u_resample;
    int32_t* out_nodes;
    int32_t* out_tokens;
    int32_t* out_n;
    double* out_log_norm;  // optional
    int32_t* out_status;   // optional
    int N, V;
    long long G;    // 16-byte groups per row
    long long GPC;  // groups per CTA of a cluster
    long long GPW;  // groups per warp (a multiple of 32)
};

// One CTA's part of a cluster exchange.
struct TreeSlot {
    double s[2];   // row sums relative to mk (target, draft), or the residual / draw sum in s[0]
    float m[2];    // row maxima, or the greedy maximum in m[0]
    float mk[2];   // integer offsets
    int bad[2];    // NaN seen
    int idx;       // greedy: first index of the maximum; draw: last index of a positive weight
    int pad;
};

// Raw bits of group g (16 / ESZ elements) of a row, -inf past V.  VEC16: the row
// is 16-byte aligned and V * ESZ a multiple of 16, so a group is one vector load;
// otherwise the elements are loaded one by one and packed the same way.
template <int ESZ, bool VEC16>
__device__ __forceinline__ uint4 tree_raw(const unsigned char* row, long long g, int V)
{
    if (VEC16) return __ldg(reinterpret_cast<const uint4*>(row) + g);
    uint32_t w[4];
    if (ESZ == 2) {
        const unsigned short* r = reinterpret_cast<const unsigned short*>(row);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const long long i = g * 8 + 2 * k;
            const uint32_t lo = i < V ? (uint32_t)__ldg(r + i) : 0xff80u;
            const uint32_t hi = i + 1 < V ? (uint32_t)__ldg(r + i + 1) : 0xff80u;
            w[k] = lo | (hi << 16);
        }
    } else {
        const uint32_t* r = reinterpret_cast<const uint32_t*>(row);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const long long i = g * 4 + k;
            w[k] = i < V ? __ldg(r + i) : 0xff800000u;
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// fp32 row state of a thread, merged across a warp.
__device__ __forceinline__ void lse_warp_merge(Lse& a)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m = __shfl_xor_sync(0xffffffffu, a.m, o);
        const float mk = __shfl_xor_sync(0xffffffffu, a.mk, o);
        const float s = __shfl_xor_sync(0xffffffffu, a.s, o);
        lse_merge(a, m, mk, s);
    }
}

// Fold (m, mk, s) parts in order into (M, MK, S) with S in fp64 relative to MK.
__device__ __forceinline__ void lse_fold64(float& M, float& MK, double& S, float m, float mk, double s)
{
    if (m == -INFINITY) return;  // an empty part (NaN is tracked apart)
    if (M == -INFINITY) {
        M = m; MK = mk; S = s;
        return;
    }
    if (mk > MK) {
        S = S * pow2d(MK - mk) + s;
        MK = mk;
    } else {
        S += s * pow2d(mk - MK);
    }
    M = fmaxf(M, m);
}

__device__ __forceinline__ void amax_warp_merge(Amax& a)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float best = __shfl_xor_sync(0xffffffffu, a.best, o);
        const int idx = __shfl_xor_sync(0xffffffffu, a.idx, o);
        const int nan = __shfl_xor_sync(0xffffffffu, a.nan, o);
        amax_merge(a, best, idx, nan);
    }
}

// Weights of one group for the residual passes and the draw: P_level(v) from p
// and q through `level` residual steps (inv_S: reciprocals of their masses), and
// w = max(0, P_level - q) when `resid` (else P_level itself).  The tests compute
// P(tok) with this same function, so both see the same bits.
struct TreeRow {
    float khi, klo, mk_t, inv_t, mk_d, inv_d;
};

__device__ __forceinline__ float tree_weight(const TreeRow& r, const float* inv_S, int level, bool resid, float lt,
                                             float ld)
{
    float P = scaled_exp(lt, r.khi, r.klo, r.mk_t) * r.inv_t;
    if (level == 0 && !resid) return P;
    const float q = scaled_exp(ld, r.khi, r.klo, r.mk_d) * r.inv_d;
    for (int k = 0; k < level; ++k) P = fmaxf(0.f, P - q) * inv_S[k];
    return resid ? fmaxf(0.f, P - q) : P;
}

// tree_weight for elements (0, 1) of a pair on packed fp32 pairs: every
// operation rounds as its scalar form in tree_weight, so both give the same bits.
__device__ __forceinline__ void tree_weight2(const TreeRow& r, const float* inv_S, int level, bool resid, float lt0,
                                             float lt1, float ld0, float ld1, float& w0, float& w1)
{
    const unsigned long long KH = pack2(r.khi, r.khi), KL = pack2(r.klo, r.klo);
    const unsigned long long xt = pack2(lt0, lt1);
    float a0, a1;
    unpack2(fma2(xt, KL, fma2(xt, KH, pack2(-r.mk_t, -r.mk_t))), a0, a1);
    unsigned long long P = mul2(pack2(ex2(a0), ex2(a1)), pack2(r.inv_t, r.inv_t));
    if (level == 0 && !resid) {
        unpack2(P, w0, w1);
        return;
    }
    const unsigned long long xd = pack2(ld0, ld1);
    float b0, b1;
    unpack2(fma2(xd, KL, fma2(xd, KH, pack2(-r.mk_d, -r.mk_d))), b0, b1);
    const unsigned long long Q = mul2(pack2(ex2(b0), ex2(b1)), pack2(r.inv_d, r.inv_d));
    for (int k = 0; k < level; ++k) {
        float d0, d1;
        unpack2(sub2(P, Q), d0, d1);
        P = mul2(pack2(fmaxf(0.f, d0), fmaxf(0.f, d1)), pack2(inv_S[k], inv_S[k]));
    }
    if (resid) {
        float d0, d1;
        unpack2(sub2(P, Q), d0, d1);
        w0 = fmaxf(0.f, d0);
        w1 = fmaxf(0.f, d1);
    } else {
        unpack2(P, w0, w1);
    }
}

// The weights of one 16-byte group (VEC elements, padded with zeros to 8).
template <int VEC>
__device__ __forceinline__ void tree_group_weights(const TreeRow& r, const float* inv_S, int level, bool resid,
                                                   const float* xt, const float* xd, float (&wv)[8])
{
#pragma unroll
    for (int e = 0; e < VEC; e += 2) tree_weight2(r, inv_S, level, resid, xt[e], xt[e + 1], xd[e], xd[e + 1], wv[e], wv[e + 1]);
#pragma unroll
    for (int e = VEC; e < 8; ++e) wv[e] = 0.f;
}

struct TreeSmem {
    TreeSlot x[2][kTreeMaxCluster];   // exchange buffers, alternating
    Lse wl[2][kTreeWarps];            // per-warp row states
    int wn[2][kTreeWarps];            // per-warp: a NaN was seen
    Amax wa[kTreeWarps];
    double wsum[kTreeWarps];
    int wlast[kTreeWarps];
    float inv_S[kTreeMaxNodes];       // residual levels of the current node
    int in[kTreeMaxNodes];            // node takes part
    int first_child[kTreeMaxNodes];
    int next_sib[kTreeMaxNodes];
    int path[kTreeMaxNodes];
    float lt[kTreeMaxNodes], ld[kTreeMaxNodes];  // the children's logits at the current node
    int pr[kTreeMaxNodes];            // the sequence's parent indices, tokens, keep flags and
    int tk[kTreeMaxNodes];            // accept uniforms, loaded once by N threads at once
    int kp[kTreeMaxNodes];
    float ua[kTreeMaxNodes];
    double lu[kTreeMaxNodes];         // log u_accept of each node
    double nn_a2[2];                  // the current node's log2-normalisers (target, draft),
    float nn_mk[2], nn_inv[2];        // offsets and reciprocal sums, folded by warp 0
    int nn_bad;
    int accept;                       // the current child's test, by thread 0
    int status;
};

// Push this CTA's slot (in `mine`) to every CTA of the cluster, then wait until
// every CTA has pushed.  `mine` is written by thread 0 before the call.
__device__ __forceinline__ void tree_exchange(cgt::cluster_group& cl, TreeSmem& sm, int par, const TreeSlot& mine,
                                             int CL, int rank)
{
    if (threadIdx.x < (unsigned)CL) *cl.map_shared_rank(&sm.x[par][rank], (int)threadIdx.x) = mine;
    cl.sync();
}

template <int ESZ, bool VEC16>
__global__ void __launch_bounds__(kTreeThreads, 2) sv_tree(TreeArgs a)
{
    constexpr int VEC = 16 / ESZ;
    __shared__ TreeSmem sm;
    __shared__ TreeSlot s_mine;
    cgt::cluster_group cl = cgt::this_cluster();
    const int CL = (int)cl.num_blocks(), rank = (int)cl.block_rank();
    const int b = (int)(blockIdx.x / (unsigned)CL);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = a.N, V = a.V;
    const size_t rowlen = (size_t)V * ESZ;
    const unsigned char* tgt = static_cast<const unsigned char*>(a.tgt) + (size_t)b * N * rowlen;
    const unsigned char* dft = static_cast<const unsigned char*>(a.dft) + (size_t)b * N * rowlen;
    const float T = a.temperature[b];
    const bool tval = temperature_ok(T), greedy = (T == 0.f);
    // this lane's groups of any row: g = lo + 32 j + lane, lo <= g < hi
    const long long cta0 = (long long)rank * a.GPC;
    const long long cta_hi = min(a.G, cta0 + a.GPC);
    const long long lo = min(cta_hi, cta0 + (long long)warp * a.GPW);
    const long long hi = min(cta_hi, lo + a.GPW);

    // ---- the tree, the nodes that take part, the input checks (every CTA alike);
    // the per-node inputs first, one node per thread, so their loads overlap
    if (tid < N) {
        const size_t i = (size_t)b * N + tid;
        sm.pr[tid] = a.parent[i];
        sm.tk[tid] = a.tokens[i];
        sm.kp[tid] = a.keep == nullptr ? 1 : a.keep[i];
        const float u = a.u_accept[i];
        sm.ua[tid] = u;
        sm.lu[tid] = log((double)u);
    }
    __syncthreads();
    const int* par = sm.pr;
    const int* tok = sm.tk;
    if (tid == 0) {
        int st = 0;
        if (!tval) st = SV_ROW_BAD_TEMPERATURE;
        if (par[0] != -1) st |= SV_ROW_BAD_TREE;
        sm.in[0] = 1;
        for (int i = 0; i < N; ++i) { sm.first_child[i] = -1; sm.next_sib[i] = -1; }
        int* last_child = sm.path;  // scratch until the walk starts
        for (int i = 0; i < N; ++i) last_child[i] = -1;
        for (int i = 1; i < N; ++i) {
            const int p = par[i];
            if (p < 0 || p >= i) { st |= SV_ROW_BAD_TREE; sm.in[i] = 0; continue; }
            sm.in[i] = sm.in[p] && sm.kp[i] != 0;
            if (!sm.in[i]) continue;
            if (tok[i] < 0 || tok[i] >= V) st |= SV_ROW_BAD_TOKEN;
            if (!greedy) {
                const float u = sm.ua[i];
                if (!(u >= 0.f && u < 1.f)) st |= SV_ROW_BAD_UNIFORM;
            }
            if (last_child[p] < 0) sm.first_child[p] = i;
            else sm.next_sib[last_child[p]] = i;
            last_child[p] = i;
        }
        if (tval && !greedy) {
            const float u = a.u_resample[b];
            if (!(u >= 0.f && u < 1.f)) st |= SV_ROW_BAD_UNIFORM;
        }
        if (!tval) st = SV_ROW_BAD_TEMPERATURE;
        sm.status = st;
    }
    if (rank == 0 && a.out_log_norm)
        for (int r = tid; r < 2 * N; r += kTreeThreads) a.out_log_norm[(size_t)b * 2 * N + r] = (double)NAN;
    cl.sync();  // every CTA runs (its shared memory exists) before any pushes to it
    int st = sm.status;

    float khi = 0.f, klo = 0.f;
    if (tval && !greedy) split_k(T, &khi, &klo);
    int c = 0, n = 0, xpar = 0, extra = -1, writer = 0;
    while (st == 0) {
        const unsigned char* trow = tgt + (size_t)c * rowlen;
        const unsigned char* drow = dft + (size_t)c * rowlen;
        const bool kids = sm.first_child[c] >= 0;
        // the children's logits at c, for the tests
        if (tid < 64) {
            int i = sm.first_child[c];
            for (int k = 0; k < tid && i >= 0; ++k) i = sm.next_sib[i];
            if (i >= 0) {
                sm.lt[tid] = load_logit<ESZ>(trow, (size_t)tok[i]);
                sm.ld[tid] = greedy ? 0.f : load_logit<ESZ>(drow, (size_t)tok[i]);
            }
        }
        if (greedy) {
            // ---- the first argmax of target row c
            Amax A{-INFINITY, 0x7fffffff, 0};
            for (long long g0 = lo + lane; g0 < hi; g0 += 32 * kTreeBatch) {
                uint4 raw[kTreeBatch];
#pragma unroll
                for (int u = 0; u < kTreeBatch; ++u)
                    if (g0 + 32 * u < hi) raw[u] = tree_raw<ESZ, VEC16>(trow, g0 + 32 * u, V);
#pragma unroll
                for (int u = 0; u < kTreeBatch; ++u)
                    if (g0 + 32 * u < hi) {
                        float x[VEC];
                        unpack<ESZ>(raw[u], x);
#pragma unroll
                        for (int e = 0; e < VEC; ++e) amax_add(A, x[e], (int)((g0 + 32 * u) * VEC + e));
                    }
            }
            amax_warp_merge(A);
            if (lane == 0) sm.wa[warp] = A;
            __syncthreads();
            if (tid == 0) {
                Amax C{-INFINITY, 0x7fffffff, 0};
                for (int w = 0; w < kTreeWarps; ++w) amax_merge(C, sm.wa[w].best, sm.wa[w].idx, sm.wa[w].nan);
                TreeSlot t{};
                t.m[0] = C.best;
                t.idx = C.idx;
                t.bad[0] = C.nan;
                s_mine = t;
            }
            __syncthreads();
            tree_exchange(cl, sm, xpar, s_mine, CL, rank);
            Amax R{-INFINITY, 0x7fffffff, 0};
            for (int r = 0; r < CL; ++r) amax_merge(R, sm.x[xpar][r].m[0], sm.x[xpar][r].idx, sm.x[xpar][r].bad[0]);
            xpar ^= 1;
            if (R.nan || R.best == INFINITY || R.best == -INFINITY) { st |= SV_ROW_BAD_LOGITS; break; }
            int next = -1, k = 0;
            for (int i = sm.first_child[c]; i >= 0; i = sm.next_sib[i], ++k)
                if (tok[i] == R.idx) { next = i; break; }
            if (next < 0) { extra = R.idx; break; }
            sm.path[n] = next;  // every CTA writes the same value
            ++n;
            c = next;
            __syncthreads();
            continue;
        }

        // ---- log-normalisers of target row c and (with children) draft row c
        Lse L[2];
        lse_init(L[0]);
        lse_init(L[1]);
        const int nrows = kids ? 2 : 1;
        for (int r = 0; r < nrows; ++r) {
            const unsigned char* row = r == 0 ? trow : drow;
            // packed fp32 pairs: one max and at most one rescale per batch, 8
            // accumulators folded at the end; groups past the part read as -inf
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            const uint32_t ninf = ESZ == 2 ? 0xff80ff80u : 0xff800000u;
            for (long long g0 = lo + lane; g0 < hi; g0 += 32 * kTreeBatch) {
                uint4 raw[kTreeBatch];
#pragma unroll
                for (int u = 0; u < kTreeBatch; ++u)
                    raw[u] = g0 + 32 * u < hi ? tree_raw<ESZ, VEC16>(row, g0 + 32 * u, V) : make_uint4(ninf, ninf, ninf, ninf);
                lse_group2<ESZ, kTreeBatch>(L[r], acc, raw, khi, klo);
            }
            lse_fold(L[r], acc);
            // a NaN anywhere makes the thread's sum NaN; it is carried apart, since a
            // part whose maximum is -inf is dropped by the merges
            const int nanf = __any_sync(0xffffffffu, L[r].s != L[r].s);
            lse_warp_merge(L[r]);
            if (lane == 0) { sm.wl[r][warp] = L[r]; sm.wn[r][warp] = nanf; }
        }
        __syncthreads();
        if (tid == 0) {
            TreeSlot t{};
            for (int r = 0; r < 2; ++r) {
                float M = -INFINITY, MK = 0.f;
                double S = 0.0;
                int nanf = 0;
                if (r < nrows)
                    for (int w = 0; w < kTreeWarps; ++w) {
                        nanf |= sm.wn[r][w];
                        lse_fold64(M, MK, S, sm.wl[r][w].m, sm.wl[r][w].mk, sm.wl[r][w].s);
                    }
                t.bad[r] = nanf;
                t.m[r] = M;
                t.mk[r] = MK;
                t.s[r] = S;
            }
            s_mine = t;
        }
        __syncthreads();
        tree_exchange(cl, sm, xpar, s_mine, CL, rank);
        // the cluster's parts folded by warp 0 (lane r: row r, parts in rank order)
        // and shared with the CTA
        if (warp == 0) {
            float Mq = -INFINITY, MKq = 0.f;
            double Sq = 0.0;
            bool bq = false;
            if (lane < nrows) {
                for (int q = 0; q < CL; ++q) {
                    bq |= sm.x[xpar][q].bad[lane] != 0;
                    lse_fold64(Mq, MKq, Sq, sm.x[xpar][q].m[lane], sm.x[xpar][q].mk[lane], sm.x[xpar][q].s[lane]);
                }
                bq |= (Mq == -INFINITY) || (Mq == INFINITY) || !isfinite(Sq) || !(Sq > 0.0);
            }
            const bool bad_any = __any_sync(0xffffffffu, bq);
            if (lane < 2) {
                const bool use = lane < nrows && !bq;
                sm.nn_a2[lane] = use ? (double)MKq + log2(Sq) : 0.0;
                sm.nn_mk[lane] = use ? MKq : 0.f;
                sm.nn_inv[lane] = use ? (float)(1.0 / Sq) : 0.f;
            }
            if (lane == 0) sm.nn_bad = bad_any;
        }
        __syncthreads();
        xpar ^= 1;
        if (sm.nn_bad) { st |= SV_ROW_BAD_LOGITS; break; }
        const double a2t = sm.nn_a2[0];
        const double a2d = kids ? sm.nn_a2[1] : 0.0;
        if (rank == 0 && tid == 0 && a.out_log_norm) {
            a.out_log_norm[(size_t)b * 2 * N + c] = a2t * kLn2;
            if (kids) a.out_log_norm[(size_t)b * 2 * N + N + c] = a2d * kLn2;
        }
        TreeRow rw;
        rw.khi = khi; rw.klo = klo;
        rw.mk_t = sm.nn_mk[0]; rw.inv_t = sm.nn_inv[0];
        rw.mk_d = kids ? sm.nn_mk[1] : 0.f; rw.inv_d = kids ? sm.nn_inv[1] : 0.f;

        // ---- the children, in index order
        const double Td = (double)T;
        int level = 0, next = -1, k = 0;
        // set when the last child's rejection applied its residual: the draw's
        // weights are that residual, so its sums (sm.wsum, sm.x[reuse_par]) stand
        int reuse_par = -1;
        for (int i = sm.first_child[c]; i >= 0; i = sm.next_sib[i], ++k) {
            // the test, by one thread for the CTA
            if (tid == 0) {
                const double lq = (double)sm.ld[k] / Td - a2d * kLn2;
                const double lp = level == 0 ? (double)sm.lt[k] / Td - a2t * kLn2
                                             : log((double)tree_weight(rw, sm.inv_S, level, false, sm.lt[k], sm.ld[k]));
                sm.accept = sm.lu[i] < lp - lq;
            }
            __syncthreads();
            if (sm.accept) { next = i; break; }
            // rejected: the mass of max(0, P - q)
            double part = 0.0;
            for (long long g0 = lo + lane; g0 < hi; g0 += 32 * kTreeBatch) {
                uint4 rt[kTreeBatch], rd[kTreeBatch];
#pragma unroll
                for (int u = 0; u < kTreeBatch; ++u)
                    if (g0 + 32 * u < hi) {
                        rt[u] = tree_raw<ESZ, VEC16>(trow, g0 + 32 * u, V);
                        rd[u] = tree_raw<ESZ, VEC16>(drow, g0 + 32 * u, V);
                    }
#pragma unroll
                for (int u = 0; u < kTreeBatch; ++u)
                    if (g0 + 32 * u < hi) {
                        float xt[VEC], xd[VEC], wv[8];
                        unpack<ESZ>(rt[u], xt);
                        unpack<ESZ>(rd[u], xd);
                        tree_group_weights<VEC>(rw, sm.inv_S, level, true, xt, xd, wv);
                        part += (double)tree8(wv);
                    }
            }
            part = warp_sum(part);
            if (lane == 0) sm.wsum[warp] = part;
            __syncthreads();
            if (tid == 0) {
                double s = 0.0;
                for (int w = 0; w < kTreeWarps; ++w) s += sm.wsum[w];
                TreeSlot t{};
                t.s[0] = s;
                s_mine = t;
            }
            __syncthreads();
            tree_exchange(cl, sm, xpar, s_mine, CL, rank);
            double S = 0.0;
            for (int q = 0; q < CL; ++q) S += sm.x[xpar][q].s[0];
            const int this_par = xpar;
            xpar ^= 1;
            if (S < kResidualMin || S != S) {
                st |= SV_ROW_RESIDUAL_ZERO;  // the residual vanished: P stays
                reuse_par = -1;
            } else {
                if (tid == 0) sm.inv_S[level] = (float)(1.0 / S);
                ++level;
                reuse_par = sm.next_sib[i] < 0 ? this_par : -1;
            }
            __syncthreads();
        }
        if (next >= 0) {
            sm.path[n] = next;
            ++n;
            c = next;
            __syncthreads();
            continue;
        }

        // ---- the extra token from P: p (no rejection) or the last residual
        const bool resid = level > 0;
        const int lev = resid ? level - 1 : 0;
        int dpar = reuse_par;
        if (dpar < 0) {
            double part = 0.0;
            for (long long g0 = lo + lane; g0 < hi; g0 += 32 * kTreeBatch) {
                uint4 rt[kTreeBatch], rd[kTreeBatch];
#pragma unroll
                for (int u = 0; u < kTreeBatch; ++u)
                    if (g0 + 32 * u < hi) {
                        rt[u] = tree_raw<ESZ, VEC16>(trow, g0 + 32 * u, V);
                        rd[u] = resid ? tree_raw<ESZ, VEC16>(drow, g0 + 32 * u, V) : rt[u];
                    }
#pragma unroll
                for (int u = 0; u < kTreeBatch; ++u)
                    if (g0 + 32 * u < hi) {
                        float xt[VEC], xd[VEC], wv[8];
                        unpack<ESZ>(rt[u], xt);
                        unpack<ESZ>(rd[u], xd);
                        tree_group_weights<VEC>(rw, sm.inv_S, lev, resid, xt, xd, wv);
                        part += (double)tree8(wv);
                    }
            }
            part = warp_sum(part);
            if (lane == 0) sm.wsum[warp] = part;
            __syncthreads();
            if (tid == 0) {
                double s = 0.0;
                for (int w = 0; w < kTreeWarps; ++w) s += sm.wsum[w];
                TreeSlot t{};
                t.s[0] = s;
                s_mine = t;
            }
            __syncthreads();
            tree_exchange(cl, sm, xpar, s_mine, CL, rank);
            dpar = xpar;
            xpar ^= 1;
        }
        double S = 0.0;
        for (int q = 0; q < CL; ++q) S += sm.x[dpar][q].s[0];
        const double target = (double)a.u_resample[b] * S;
        // the last token of this CTA's range with a positive weight (-1 if none):
        // only for the rare draw that rounding leaves without a crossing
        auto cta_last_positive = [&]() -> int {
            int last = -1;
            for (long long g = lo + lane; g < hi; g += 32) {
                float xt[VEC], xd[VEC];
                const uint4 rt = tree_raw<ESZ, VEC16>(trow, g, V);
                unpack<ESZ>(rt, xt);
                unpack<ESZ>(resid ? tree_raw<ESZ, VEC16>(drow, g, V) : rt, xd);
#pragma unroll
                for (int e = 0; e < VEC; ++e)
                    if (tree_weight(rw, sm.inv_S, lev, resid, xt[e], xd[e]) > 0.f) last = (int)(g * VEC + e);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
            if (lane == 0) sm.wlast[warp] = last;
            __syncthreads();
            int l = -1;
            for (int w = 0; w < kTreeWarps; ++w) l = max(l, sm.wlast[w]);
            __syncthreads();
            return l;
        };
        // the CTA whose range holds the crossing
        int rstar = -1;
        double before = 0.0;
        {
            double C = 0.0;
            for (int q = 0; q < CL; ++q) {
                const double s = sm.x[dpar][q].s[0];
                if (C + s > target) { rstar = q; before = C; break; }
                C += s;
            }
        }
        writer = rstar >= 0 ? rstar : 0;
        if (rstar < 0) {
            // rounding left no crossing: the last token with a positive weight
            // over the whole row (every CTA of the cluster takes this branch)
            const int l = cta_last_positive();
            if (tid == 0) {
                TreeSlot t{};
                t.idx = l;
                s_mine = t;
            }
            __syncthreads();
            tree_exchange(cl, sm, xpar, s_mine, CL, rank);
            int lastpos = -1;
            for (int q = 0; q < CL; ++q) lastpos = max(lastpos, sm.x[xpar][q].idx);
            xpar ^= 1;
            extra = lastpos;
        }
        if (rstar == rank) {
            // warp holding the crossing, then its 32-group blocks, lanes and elements
            __shared__ int s_found;
            if (tid == 0) {
                int ws = -1;
                double C = before;
                for (int w = 0; w < kTreeWarps; ++w) {
                    if (C + sm.wsum[w] > target) { ws = w; before = C; break; }
                    C += sm.wsum[w];
                }
                s_found = ws;
                sm.wsum[0] = before;  // the mass before warp ws
            }
            __syncthreads();
            const int ws = s_found;
            int tokf = -1;
            if (ws >= 0 && warp == ws) {
                // the warp's groups into L1 first (from L2, where the passes left
                // them), so the walk below does not wait on L2 once per block
                if constexpr (VEC16) {
                    for (long long g = lo + lane; g < hi; g += 32) {
                        asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<const uint4*>(trow) + g));
                        if (resid) asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<const uint4*>(drow) + g));
                    }
                }
                double C = sm.wsum[0];
                for (long long gb = lo; gb < hi && tokf < 0; gb += 32) {
                    const long long g = gb + lane;
                    float wv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) wv[e] = 0.f;
                    if (g < hi) {
                        float xt[VEC], xd[VEC];
                        const uint4 rt = tree_raw<ESZ, VEC16>(trow, g, V);
                        unpack<ESZ>(rt, xt);
                        unpack<ESZ>(resid ? tree_raw<ESZ, VEC16>(drow, g, V) : rt, xd);
#pragma unroll
                        for (int e = 0; e < VEC; ++e) wv[e] = tree_weight(rw, sm.inv_S, lev, resid, xt[e], xd[e]);
                    }
                    const double mine = (double)tree8(wv);
                    const double incl = warp_inclusive_scan(mine);
                    const double tot = __shfl_sync(0xffffffffu, incl, 31);
                    if (C + tot > target) {
                        const unsigned hit = __ballot_sync(0xffffffffu, C + incl > target);
                        const int ls = __ffs(hit) - 1;
                        if (lane == ls) {
                            double E = C + incl - mine;
                            int kk = -1, lastv = -1;
                            for (int e = 0; e < VEC; ++e) {
                                if (wv[e] > 0.f) lastv = e;
                                E += (double)wv[e];
                                if (E > target && wv[e] > 0.f) { kk = e; break; }
                            }
                            if (kk < 0) kk = lastv >= 0 ? lastv : 0;
                            tokf = (int)(g * VEC + kk);
                        }
                        tokf = __shfl_sync(0xffffffffu, tokf, ls);
                        break;
                    }
                    C += tot;
                }
                if (lane == 0 && tokf >= 0) s_found = -2 - tokf;
            }
            __syncthreads();
            if (s_found <= -2) extra = -2 - s_found;
            else extra = cta_last_positive();  // the search lost the crossing to rounding
        }
        break;
    }

    // ---- outputs, from one CTA: the one that found the extra token (rank 0 on
    // errors, for greedy sequences, and when rounding left no crossing)
    if (rank == writer) {
        const bool bad = (st & (SV_ROW_BAD_TOKEN | SV_ROW_BAD_LOGITS | SV_ROW_BAD_TEMPERATURE | SV_ROW_BAD_UNIFORM |
                                SV_ROW_BAD_TREE)) != 0;
        const int nn = bad ? 0 : n;
        int32_t* on = a.out_nodes + (size_t)b * N;
        int32_t* ot = a.out_tokens + (size_t)b * N;
        for (int j = tid; j < N; j += kTreeThreads) {
            on[j] = (!bad && j < nn) ? sm.path[j] : -1;
            ot[j] = bad ? -1 : (j < nn ? tok[sm.path[j]] : (j == nn ? extra : -1));
        }
        if (tid == 0) {
            a.out_n[b] = nn;
            if (a.out_status) a.out_status[b] = st;
        }
    }
    cl.sync();  // no CTA leaves while another may still push to its shared memory
}

// ---------------------------------------------------------------------------- pruning

struct PruneArgs {
    const void* dft;
    const int32_t* parent;
    const int32_t* tokens;
    const float* temperature;
    double threshold;
    int32_t* out_keep;
    double* out_cum;  // first the draft log-probabilities of the nodes, then their sums
    int B, N, V;
    long long G;
};

// A sequence takes part in pruning when its temperature is valid, parent[0] = -1
// and 0 <= parent[i] < i for every other node (each lane checks its nodes).
__device__ __forceinline__ bool prune_node_ok(int i, int p) { return i == 0 ? p == -1 : (p >= 0 && p < i); }

// One CTA per (sequence b, node c) of a well-formed sequence in which c has
// children: log q_c(tok_i) for every child i of c -- ld/T - lse(ld/T) of draft row
// c (T > 0), or 0 / -inf as tok_i is / is not the first argmax of that row (T = 0);
// NaN for a token outside [0, V) or a bad row.
template <int ESZ, bool VEC16>
__global__ void __launch_bounds__(kPruneThreads) sv_tree_prune_rows(PruneArgs a)
{
    constexpr int VEC = 16 / ESZ;
    constexpr int NW = kPruneThreads / 32;
    __shared__ int s_go;
    __shared__ Lse s_l[NW];
    __shared__ int s_n[NW];
    __shared__ Amax s_a[NW];
    __shared__ double s_lse;
    __shared__ int s_arg, s_bad;
    const int b = (int)(blockIdx.x / (unsigned)a.N), c = (int)(blockIdx.x % (unsigned)a.N);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t* par = a.parent + (size_t)b * a.N;
    const int32_t* tok = a.tokens + (size_t)b * a.N;
    const float T = a.temperature[b];
    if (warp == 0) {
        // the sequence's tree is well formed and c has a child: one parent index
        // per lane, all loads in flight at once
        bool ok = temperature_ok(T), kid = false;
        for (int i = lane; i < a.N; i += 32) {
            const int p = par[i];
            ok = ok && prune_node_ok(i, p);
            kid = kid || (i > c && p == c);
        }
        ok = __all_sync(0xffffffffu, ok);
        kid = __any_sync(0xffffffffu, kid);
        if (lane == 0) s_go = ok && kid;
    }
    __syncthreads();
    if (!s_go) return;
    const bool greedy = (T == 0.f);
    float khi = 0.f, klo = 0.f;
    if (!greedy) split_k(T, &khi, &klo);
    const unsigned char* row = static_cast<const unsigned char*>(a.dft) + ((size_t)b * a.N + c) * (size_t)a.V * ESZ;
    Lse L;
    lse_init(L);
    Amax A{-INFINITY, 0x7fffffff, 0};
    constexpr int kPB = 4;  // groups per thread loaded before any is used
    // the normaliser on packed fp32 pairs (one max and at most one rescale per
    // batch, 8 accumulators folded at the end); groups past the row read as -inf
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const uint32_t ninf = ESZ == 2 ? 0xff80ff80u : 0xff800000u;
    for (long long g0 = tid; g0 < a.G; g0 += (long long)kPruneThreads * kPB) {
        uint4 raw[kPB];
#pragma unroll
        for (int u = 0; u < kPB; ++u) {
            const long long g = g0 + (long long)kPruneThreads * u;
            raw[u] = g < a.G ? tree_raw<ESZ, VEC16>(row, g, a.V) : make_uint4(ninf, ninf, ninf, ninf);
        }
        if (greedy) {
#pragma unroll
            for (int u = 0; u < kPB; ++u) {
                const long long g = g0 + (long long)kPruneThreads * u;
                if (g >= a.G) break;
                float x[VEC];
                unpack<ESZ>(raw[u], x);
#pragma unroll
                for (int e = 0; e < VEC; ++e) amax_add(A, x[e], (int)(g * VEC + e));
            }
        } else {
            lse_group2<ESZ, kPB>(L, acc, raw, khi, klo);
        }
    }
    if (!greedy) lse_fold(L, acc);
    const int nanf = __any_sync(0xffffffffu, L.s != L.s);
    lse_warp_merge(L);
    amax_warp_merge(A);
    if (lane == 0) { s_l[warp] = L; s_n[warp] = nanf; s_a[warp] = A; }
    __syncthreads();
    if (tid == 0) {
        if (greedy) {
            Amax C{-INFINITY, 0x7fffffff, 0};
            for (int w = 0; w < NW; ++w) amax_merge(C, s_a[w].best, s_a[w].idx, s_a[w].nan);
            s_arg = C.idx;
            s_bad = C.nan || C.best == INFINITY || C.best == -INFINITY;
        } else {
            float M = -INFINITY, MK = 0.f;
            double S = 0.0;
            int bad = 0;
            for (int w = 0; w < NW; ++w) {
                bad |= s_n[w];
                lse_fold64(M, MK, S, s_l[w].m, s_l[w].mk, s_l[w].s);
            }
            bad |= (M == -INFINITY) || (M == INFINITY) || !isfinite(S) || !(S > 0.0);
            s_bad = bad;
            s_lse = ((double)MK + log2(S)) * kLn2;
        }
    }
    __syncthreads();
    for (int i = c + 1 + tid; i < a.N; i += kPruneThreads) {
        if (par[i] != c) continue;
        const int x = tok[i];
        double lq = NAN;
        if (x >= 0 && x < a.V && !s_bad)
            lq = greedy ? (x == s_arg ? 0.0 : -INFINITY) : (double)load_logit<ESZ>(row, (size_t)x) / (double)T - s_lse;
        a.out_cum[(size_t)b * a.N + i] = lq;
    }
}

// One warp per sequence: cum[i] = cum[parent] + log q, keep[i] = keep[parent]
// and not (cum[i] < threshold), in node order (parents come first).  The parents
// and log-probabilities are loaded by the lanes at once and walked in shared
// memory by lane 0.  A sequence with a bad temperature or tree keeps every node,
// with cum NaN.
constexpr int kWalkWarps = 4;

__global__ void __launch_bounds__(kWalkWarps * 32) sv_tree_prune_walk(PruneArgs a)
{
    __shared__ double s_cum[kWalkWarps][kTreeMaxNodes];
    __shared__ int s_par[kWalkWarps][kTreeMaxNodes];
    __shared__ int s_keep[kWalkWarps][kTreeMaxNodes];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = (int)blockIdx.x * kWalkWarps + warp;
    if (b >= a.B) return;  // the whole warp
    const int N = a.N;
    const int32_t* par = a.parent + (size_t)b * N;
    double* cum = a.out_cum + (size_t)b * N;
    int32_t* keep = a.out_keep + (size_t)b * N;
    bool ok = temperature_ok(a.temperature[b]);
    for (int i = lane; i < N; i += 32) {
        const int p = par[i];
        s_par[warp][i] = p;
        s_cum[warp][i] = cum[i];
        ok = ok && prune_node_ok(i, p);
    }
    if (!__all_sync(0xffffffffu, ok)) {
        for (int i = lane; i < N; i += 32) { keep[i] = 1; cum[i] = (double)NAN; }
        return;
    }
    __syncwarp();
    if (lane == 0) {
        double* sc = s_cum[warp];
        int* sk = s_keep[warp];
        const int* sp = s_par[warp];
        sc[0] = 0.0;
        sk[0] = 1;
        for (int i = 1; i < N; ++i) {
            const int c = sp[i];
            sc[i] = sc[c] + sc[i];
            sk[i] = sk[c] && !(sc[i] < a.threshold);
        }
    }
    __syncwarp();
    for (int i = lane; i < N; i += 32) {
        cum[i] = s_cum[warp][i];
        keep[i] = s_keep[warp][i];
    }
}

}  // namespace sv
