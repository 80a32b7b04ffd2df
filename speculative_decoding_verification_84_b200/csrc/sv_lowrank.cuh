// sv_lowrank.cuh -- the low-rank draft head on the 5th-generation tensor cores
// [SlimSpec, Metodologia, "Arquitetura": z = W_up W_down h, W_down in R^{r x d},
// W_up in R^{V x r}, r << d, in place of the full-rank z = W_full h].
//
// Both contractions are out = A B^T with A [rows][K] and B [cols][K] bf16,
// K-major (the layout of h, W_down and W_up as stored), fp32 accumulation:
//   down:  u [M][r] = h [M][d]  W_down [r][d]^T   (rounded to bf16: the second
//          contraction takes bf16 operands)
//   up:    z [M][V] = u [M][r]  W_up [V][r]^T     (bf16 logits for the verifier)
// and the up contraction's epilogue also folds each row's online log-sum-exp of
// its bf16 logits at the row's temperature (the draft row's normaliser, the
// arithmetic of the verifier's passes), written as one partial per (row,
// column tile) and folded by sv_lr_lse.
//
// sv_lr_gemm: persistent, one CTA per SM walking 128 x BN output tiles, the
// accumulator double-buffered in TMEM.  When K fits (K <= 512, the up contraction
// with r <= 512), a CTA keeps one row tile of A (all of K) in shared memory and
// streams only B; the CTAs of a slot walk the same column tiles, so each W tile
// comes from HBM once.  Otherwise both operands stream through the ring.
//   warp 0 (one thread)  TMA: 128 x 64 of A and BN x 64 of B per stage, 128-byte
//                        swizzle, kLrStages stages, mbarrier transaction counts
//   warp 1 (one thread)  tcgen05.mma kind::f16 (bf16 x bf16 -> f32), M = 128,
//                        N = BN, four K = 16 steps per stage, accumulator in
//                        TMEM; tcgen05.commit frees the stage, and after the last
//                        stage signals the epilogue
//   warp 2               allocates and frees the TMEM columns
//   warps 4-11           epilogue: tcgen05.ld of 32 lanes x 32 columns at a
//                        time (warp 4 + w reads lanes 32 (w % 4) ... + 31 and the
//                        columns of group w / 4), bf16 rounding, 16-byte stores,
//                        the row's online log-sum-exp over its group
// Every wait on an mbarrier is bounded: past kLrPolls polls the CTA raises
// *err, stops issuing, and still frees its TMEM.
#pragma once

#include <cuda.h>  // CUtensorMap
#include <cuda_bf16.h>

#include "sv_common.cuh"

namespace sv {

constexpr int kLrBM = 128;      // tile rows = the MMA's M
constexpr int kLrBK = 64;       // K per stage: one 128-byte swizzled row of bf16
constexpr int kLrMaxStages = 4;
constexpr int kLrMaxResidentKb = 8;  // A stays in shared memory when K <= 8 x 64
constexpr int kLrEpiWarps = 8;   // per TMEM lane quarter kLrGroups warps, each on a column group
constexpr int kLrGroups = kLrEpiWarps / 4;
constexpr int kLrThreads = 128 + 32 * kLrEpiWarps;
constexpr int kLrSmemMax = 227 * 1024 - 1024;  // dynamic shared memory of one CTA (static part kept apart)

struct LrArgs {
    __nv_bfloat16* out;        // [M][N]
    float4* part;              // [M][kLrGroups n_tiles] (m, mk, s, 0) per column group, or null
    const float* temperature;  // [M] or null (T = 1)
    int* err;                  // optional: 1 if a wait gave up
    int M, N, K;
    int m_tiles, n_tiles;
    int stages;                // ring depth
    int a_resident;            // the CTA's A tile (all of K) is loaded once and kept
    int tma_store;             // out written by TMA stores of 32 x 32 chunks staged in shared memory
    int splits;                // K split this many ways (no A residency, no normaliser): each
    float* part_out;           // slice writes fp32 [splits][M][N] here, summed by sv_lr_splitk_sum
};

constexpr int kLrChunkBytes = 32 * 32 * 2;                      // one 32-row x 32-column bf16 chunk
constexpr int kLrStagingBytes = kLrEpiWarps * 2 * kLrChunkBytes;  // two chunks per epilogue warp

__device__ __forceinline__ uint32_t lr_smem(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void lr_mbar_init(uint64_t* bar, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(lr_smem(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void lr_expect_tx(uint64_t* bar, unsigned bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(lr_smem(bar)), "r"(bytes) : "memory");
}

// One poll that may suspend the thread for up to kLrPollNs while the phase is
// still open (it returns as soon as the phase completes), so waiting warps take
// no issue slots from the producer and the MMA thread.
constexpr unsigned kLrPollNs = 20000;
constexpr unsigned kLrPolls = 200000;  // with the suspension: seconds, not hours

__device__ __forceinline__ bool lr_try_wait(uint64_t* bar, unsigned parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(lr_smem(bar)), "r"(parity), "r"(kLrPollNs)
        : "memory");
    return ok != 0;
}

// Wait for the phase with this parity; false (after raising the flags) if it did
// not complete within kLrPolls polls, or another role of the CTA already gave up.
__device__ __forceinline__ bool lr_wait(uint64_t* bar, unsigned parity, volatile int* abort, int* err)
{
    for (unsigned i = 0; i < kLrPolls; ++i) {
        if (lr_try_wait(bar, parity)) return true;
        if ((i & 63u) == 63u && *abort) return false;
    }
    *abort = 1;
    if (err) atomicExch(err, 1);
    return false;
}

// shared -> global tensor store of one staged chunk; rows and columns past the
// tensor's extent are not written
__device__ __forceinline__ void lr_tma_store_2d(const CUtensorMap* map, const void* src, int x, int y)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"((uint64_t)map),
                 "r"(lr_smem(src)), "r"(x), "r"(y)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void lr_tma_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            lr_smem(dst)),
        "l"((uint64_t)map), "r"(lr_smem(bar)), "r"(x), "r"(y)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t lr_desc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu)   // start address, 16-byte units
           | ((uint64_t)1 << 16)                 // leading byte offset (unused for swizzled K-major)
           | ((uint64_t)(1024 >> 4) << 32)       // stride byte offset: 8 rows x 128 bytes
           | ((uint64_t)1 << 46)                 // descriptor version (sm_100)
           | ((uint64_t)2 << 61);                // layout: 128-byte swizzle
}

// Instruction descriptor: f32 accumulator, bf16 A and B, both K-major, M x N.
template <int N>
__device__ __forceinline__ constexpr uint32_t lr_idesc()
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kLrBM >> 4) << 24);
}

__device__ __forceinline__ void lr_mma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

__device__ __forceinline__ void lr_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(lr_smem(bar))
                 : "memory");
}

__device__ __forceinline__ void lr_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void lr_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void lr_tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void lr_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(lr_smem(bar)) : "memory");
}

// The k-th tile of CTA c, or false past its last.  A resident: the CTA keeps
// row tile c % m_tiles and walks column tiles slot, slot + nslots, ... (the
// CTAs of one slot run the same column tile at about the same time, so its W
// rows come from HBM once); otherwise tiles c, c + gridDim.x, ... with the row
// tile fastest.
__device__ __forceinline__ bool lr_tile(const LrArgs& g, int k, int* m, int* n, int* ks)
{
    *ks = 0;
    if (g.a_resident) {
        const int nslots = (int)gridDim.x / g.m_tiles;
        *m = (int)blockIdx.x % g.m_tiles;
        *n = (int)blockIdx.x / g.m_tiles + k * nslots;
        return *n < g.n_tiles;
    }
    const long long t = (long long)blockIdx.x + (long long)k * gridDim.x;
    if (t >= (long long)g.m_tiles * g.n_tiles * g.splits) return false;
    *m = (int)(t % g.m_tiles);
    const long long rest = t / g.m_tiles;
    *n = (int)(rest % g.n_tiles);
    *ks = (int)(rest / g.n_tiles);
    return true;
}

// K blocks [kb0, kb1) of slice ks.
__device__ __forceinline__ void lr_kslice(const LrArgs& g, int kbs, int ks, int* kb0, int* kb1)
{
    const int per = (kbs + g.splits - 1) / g.splits;
    *kb0 = min(kbs, ks * per);
    *kb1 = min(kbs, *kb0 + per);
}

// Persistent, one CTA per SM; the accumulator is double-buffered in TMEM (2 x BN
// columns): while the epilogue warps drain tile i from one buffer, the MMA thread
// fills the other with tile i + 1, and the producer keeps loading ahead through
// the stage ring.
template <int BN>
__global__ void __launch_bounds__(kLrThreads, 1)
    sv_lr_gemm(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
               const __grid_constant__ CUtensorMap tc, LrArgs g)
{
    static_assert(BN == 32 || BN == 64 || BN == 128 || BN == 256, "tile columns: a power of two TMEM allocation");
    constexpr int A_BYTES = kLrBM * kLrBK * 2;  // one K block of A
    constexpr int B_BYTES = BN * kLrBK * 2;
    constexpr uint32_t kCols = 2 * BN;          // two accumulators
    extern __shared__ unsigned char lr_dyn[];
    // every tile starts on a 1024-byte boundary of the shared window (the swizzle atom)
    unsigned char* sm = lr_dyn + ((1024u - (lr_smem(lr_dyn) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t full[kLrMaxStages], empty[kLrMaxStages], tfull[2], tempty[2], afull;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort, s_consumed, s_a_done;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kbs = (g.K + kLrBK - 1) / kLrBK;
    const bool res = g.a_resident != 0;
    const int S = g.stages;
    const int STAGE = res ? B_BYTES : A_BYTES + B_BYTES;
    unsigned char* ring = sm + (res ? kbs * A_BYTES : 0);
    unsigned char* staging = ring + S * STAGE;  // tma_store: kLrStagingBytes after the ring

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            lr_mbar_init(&full[s], 1);
            lr_mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            lr_mbar_init(&tfull[b], 1);
            lr_mbar_init(&tempty[b], kLrEpiWarps);  // one arrival per epilogue warp
        }
        lr_mbar_init(&afull, 1);
        s_abort = 0;
        s_consumed = 0;
        s_a_done = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(lr_smem(&s_tmem)),
                     "r"(kCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    lr_fence_before();
    __syncthreads();
    lr_fence_after();
    const uint32_t tmem = s_tmem;
    volatile int* abort = &s_abort;

    int issued = 0, a_issued = 0;
    if (warp == 0 && lane == 0) {
        // ---- producer: one global count of stages across the CTA's tiles
        int m0, n0, k0;
        if (res && lr_tile(g, 0, &m0, &n0, &k0)) {
            lr_expect_tx(&afull, (unsigned)(kbs * A_BYTES));
            for (int kb = 0; kb < kbs; ++kb) lr_tma_2d(sm + kb * A_BYTES, &ta, &afull, kb * kLrBK, m0 * kLrBM);
            a_issued = 1;
        }
        int it = 0, m, n, ks;
        bool ok = true;
        for (int k = 0; ok && lr_tile(g, k, &m, &n, &ks); ++k) {
            int kb0, kb1;
            lr_kslice(g, kbs, ks, &kb0, &kb1);
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int s = it % S;
                const unsigned ph = (unsigned)(it / S);
                if (it >= S && !lr_wait(&empty[s], (ph - 1u) & 1u, abort, g.err)) { ok = false; break; }
                unsigned char* st = ring + s * STAGE;
                lr_expect_tx(&full[s], (unsigned)STAGE);
                if (!res) lr_tma_2d(st, &ta, &full[s], kb * kLrBK, m * kLrBM);
                lr_tma_2d(st + (res ? 0 : A_BYTES), &tb, &full[s], kb * kLrBK, n * BN);
                issued = it + 1;
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer
        constexpr uint32_t idesc = lr_idesc<BN>();
        int it = 0, i = 0, m, n, ks;
        bool ok = true;
        if (res && lr_tile(g, 0, &m, &n, &ks)) {
            ok = lr_wait(&afull, 0u, abort, g.err);
            s_a_done = ok ? 1 : 0;
        }
        for (; ok && lr_tile(g, i, &m, &n, &ks); ++i) {
            const int b = i & 1, use = i >> 1;
            if (use >= 1 && !lr_wait(&tempty[b], (unsigned)(use - 1) & 1u, abort, g.err)) break;
            lr_fence_after();
            const uint32_t d = tmem + (uint32_t)(b * BN);
            int kb0, kb1;
            lr_kslice(g, kbs, ks, &kb0, &kb1);
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int s = it % S;
                const unsigned ph = (unsigned)(it / S);
                if (!lr_wait(&full[s], ph & 1u, abort, g.err)) { ok = false; break; }
                lr_fence_after();
                const uint32_t st = lr_smem(ring + s * STAGE);
                const uint32_t a0 = res ? lr_smem(sm + kb * A_BYTES) : st;
                const uint32_t b0 = res ? st : st + A_BYTES;
#pragma unroll
                for (int j = 0; j < kLrBK / 16; ++j)  // K = 16 per MMA: 32 bytes along the swizzled row
                    lr_mma(d, lr_desc(a0 + 32 * j), lr_desc(b0 + 32 * j), idesc, (kb > kb0 || j > 0) ? 1u : 0u);
                lr_commit(&empty[s]);
                s_consumed = it + 1;
            }
            lr_commit(&tfull[b]);
        }
    } else if (warp >= 4) {
        // ---- epilogue: warp 4 + w owns TMEM lanes (= tile rows) 32q .. 32q + 31,
        // q = w % 4, and column group w / 4 (QCOLS columns; a tcgen05.ld reads 32, so
        // with BN < 128 the groups past BN read nothing but still wait for and hand
        // back each accumulator: the barrier counts every epilogue warp)
        const int q = (warp - 4) & 3, grp = (warp - 4) >> 2;
        constexpr int QCOLS = BN / kLrGroups >= 32 ? BN / kLrGroups : 32;
        const bool active = grp * QCOLS < BN;
        const bool lse = g.part != nullptr;
        unsigned char* stg = staging + (warp - 4) * 2 * kLrChunkBytes;
        int chunks = 0;  // chunks this warp has staged (the buffer alternates)
        int i = 0, m_tile, n_tile, ks;
        for (; lr_tile(g, i, &m_tile, &n_tile, &ks); ++i) {
            const int b = i & 1, use = i >> 1;
            const int row = m_tile * kLrBM + 32 * q + lane;
            const bool row_ok = row < g.M;
            float4* part = (lse && row_ok) ? g.part + ((size_t)row * g.n_tiles + n_tile) * kLrGroups + grp : nullptr;
            // one lane waits, so the warp-wide tcgen05.ld below runs on all lanes or none
            int ready = 0;
            if (lane == 0) ready = lr_wait(&tfull[b], (unsigned)use & 1u, abort, g.err) ? 1 : 0;
            ready = __shfl_sync(0xffffffffu, ready, 0);
            if (!ready) break;
            lr_fence_after();
            if (!active) {
                __syncwarp();
                if (lane == 0) lr_arrive(&tempty[b]);
                if (part) *part = make_float4(-INFINITY, 0.f, 0.f, 0.f);
                continue;
            }
            float T = 1.f;
            if (part && g.temperature) T = g.temperature[row];
            const bool lse_row = part != nullptr && T > 0.f && T <= FLT_MAX;
            float khi = 0.f, klo = 0.f;
            if (lse_row) split_k(T, &khi, &klo);
            Lse L;
            lse_init(L);
            const uint32_t tb_addr = tmem + (uint32_t)(b * BN + grp * QCOLS) + ((uint32_t)(32 * q) << 16);
            for (int c = 0; c < QCOLS; c += 32) {
                uint32_t r[32];
                lr_tmem_ld32(tb_addr + (uint32_t)c, r);
                if (c + 32 == QCOLS) {
                    // this warp's part of the accumulator is read: hand it back
                    lr_fence_before();
                    __syncwarp();
                    if (lane == 0) lr_arrive(&tempty[b]);
                }
                const int n0 = n_tile * BN + grp * QCOLS + c;
                if (g.splits > 1) {
                    // a K slice: the raw fp32 sums, for sv_lr_splitk_sum
                    if (row_ok) {
                        float* dst = g.part_out + ((size_t)ks * g.M + row) * g.N + n0;
                        if (n0 + 32 <= g.N && (g.N & 3) == 0) {
#pragma unroll
                            for (int v = 0; v < 8; ++v)
                                reinterpret_cast<uint4*>(dst)[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
                        } else {
#pragma unroll
                            for (int k = 0; k < 32; ++k)  // unrolled: r stays in registers
                                if (n0 + k < g.N) dst[k] = __uint_as_float(r[k]);
                        }
                    }
                    continue;
                }
                float x[32];
                uint32_t packed[16];
#pragma unroll
                for (int k = 0; k < 32; k += 2) {
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[k]), __uint_as_float(r[k + 1]));
                    packed[k / 2] = *reinterpret_cast<const uint32_t*>(&h2);
                    x[k] = __bfloat162float(h2.x);
                    x[k + 1] = __bfloat162float(h2.y);
                }
                if (g.tma_store) {
                    // stage the warp's 32 x 32 chunk (lane = row, 64 bytes each) and
                    // let one TMA store write it
                    unsigned char* buf = stg + (chunks & 1) * kLrChunkBytes;
                    if (chunks >= 2) {
                        if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                        __syncwarp();
                    }
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        reinterpret_cast<uint4*>(buf + lane * 64)[v] =
                            make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) lr_tma_store_2d(&tc, buf, n0, m_tile * kLrBM + 32 * q);
                    ++chunks;
                } else if (row_ok) {
                    __nv_bfloat16* dst = g.out + (size_t)row * g.N + n0;
                    if (n0 + 32 <= g.N && (g.N & 7) == 0) {
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            reinterpret_cast<uint4*>(dst)[v] =
                                make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                    } else {
#pragma unroll
                        for (int k = 0; k < 32; ++k)  // unrolled: packed stays in registers
                            if (n0 + k < g.N)
                                reinterpret_cast<unsigned short*>(dst)[k] =
                                    (unsigned short)((k & 1) ? (packed[k / 2] >> 16) : (packed[k / 2] & 0xffffu));
                    }
                }
                if (lse_row) {
                    // one maximum and at most one rescale per 32 columns, then 32
                    // independent terms on packed fp32 pairs (each term rounds as
                    // scaled_exp's), columns past N only in the last column tile
                    if (n0 + 32 > g.N) {
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            if (n0 + k >= g.N) x[k] = -INFINITY;
                    }
                    float vm = x[0];
#pragma unroll
                    for (int k = 1; k < 32; ++k) vm = fmaxf(vm, x[k]);
                    lse_rebase(L, vm, khi);
                    const unsigned long long KH = pack2(khi, khi), KL = pack2(klo, klo), NM = pack2(-L.mk, -L.mk);
                    unsigned long long acc2[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc2[e] = pack2(0.f, 0.f);
#pragma unroll
                    for (int k = 0; k < 32; k += 2) {
                        const unsigned long long x2 = pack2(x[k], x[k + 1]);
                        const unsigned long long y2 = fma2(x2, KL, fma2(x2, KH, NM));
                        float y0, y1;
                        unpack2(y2, y0, y1);
                        acc2[(k >> 1) & 3] = add2(acc2[(k >> 1) & 3], pack2(ex2(y0), ex2(y1)));
                    }
                    float acc[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) unpack2(acc2[e], acc[2 * e], acc[2 * e + 1]);
                    L.s += tree8(acc);
                }
            }
            if (part) *part = make_float4(L.m, L.mk, L.s, 0.f);
        }
        // the staged chunks are written before the CTA (and its shared memory) ends
        if (g.tma_store && lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        __syncwarp();
    }
    lr_fence_before();
    __syncthreads();
    // after a wait gave up: let the copies this CTA issued but never consumed land
    // (bounded) before its shared memory goes away
    if (warp == 0 && lane == 0 && s_abort) {
        if (a_issued && !s_a_done)
            for (unsigned k = 0; k < kLrPolls && !lr_try_wait(&afull, 0u); ++k) {
            }
        for (int it = s_consumed; it < issued; ++it) {
            const unsigned par = (unsigned)(it / S) & 1u;
            for (unsigned k = 0; k < kLrPolls && !lr_try_wait(&full[it % S], par); ++k) {
            }
        }
    }
    if (warp == 2) {
        lr_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols));
    }
}

// out [M][N] = bf16 of the sum of the K slices' fp32 partials, slice 0 first.
__global__ void sv_lr_splitk_sum(const float* __restrict__ part, int splits, int M, int N,
                                 __nv_bfloat16* __restrict__ out)
{
    const long long total = (long long)M * N;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        float acc = part[i];
        for (int s = 1; s < splits; ++s) acc += part[(long long)s * total + i];
        out[i] = __float2bfloat16_rn(acc);
    }
}

// One warp per row: fold the row's column-tile partials into lse = (MK + log2 S) ln 2
// (NaN for T = 0, an invalid T, or a row with NaN or +inf).
__global__ void sv_lr_lse(const float4* __restrict__ part, const float* __restrict__ temperature, int M, int n_tiles,
                          double* __restrict__ out_lse)
{
    const int row = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (row >= M) return;
    const float T = temperature ? temperature[row] : 1.f;
    float M_ = -INFINITY, MK = 0.f;
    double S = 0.0;
    int nan = 0;
    for (int t = lane; t < n_tiles; t += 32) {
        const float4 p = part[(size_t)row * n_tiles + t];
        nan |= (p.z != p.z);
        if (p.x == -INFINITY) continue;
        if (M_ == -INFINITY) { M_ = p.x; MK = p.y; S = (double)p.z; continue; }
        if (p.y > MK) { S = S * pow2d(MK - p.y) + (double)p.z; MK = p.y; }
        else S += (double)p.z * pow2d(p.y - MK);
        M_ = fmaxf(M_, p.x);
    }
    // fold the lanes (xor tree: every lane ends with the same values)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, M_, o);
        const float mk2 = __shfl_xor_sync(0xffffffffu, MK, o);
        const double s2 = __shfl_xor_sync(0xffffffffu, S, o);
        nan |= __shfl_xor_sync(0xffffffffu, nan, o);
        if (m2 == -INFINITY) continue;
        if (M_ == -INFINITY) { M_ = m2; MK = mk2; S = s2; continue; }
        if (mk2 > MK) { S = S * pow2d(MK - mk2) + s2; MK = mk2; }
        else S += s2 * pow2d(mk2 - MK);
        M_ = fmaxf(M_, m2);
    }
    if (lane == 0) {
        const bool ok = T > 0.f && T <= FLT_MAX && !nan && M_ != -INFINITY && M_ != INFINITY && S > 0.0 && S <= DBL_MAX;
        out_lse[row] = ok ? ((double)MK + log2(S)) * kLn2 : (double)NAN;
    }
}

}  // namespace sv
