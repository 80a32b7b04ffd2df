// sv_stream.cuh -- the streaming path: one persistent, warp-specialised CTA per SM.
//
// Work list.  Item i of a call is decoded from i alone.  Items come in
// super-steps s = 0 .. B+D-1; super-step s holds
//   * the R*nI1 row-segment items of sequence s (pass 1: normaliser partials), then
//   * the nI2 residual items of sequence s-D (pass 2: residual / bonus weight sums).
// The delay D (in sequences) makes the residual rows of a sequence get re-read
// while they are still in L2, after its pass 1 has had time to finish.
//
// Roles inside a CTA (20 warps):
//   consumers (warps 0-15) two groups of 8 warps take alternate items (ping-pong:
//                          one group's reductions overlap the other's exponentials),
//                          read the item's stage of a kStages-deep shared-memory
//                          ring, free it (one "empty" arrival per warp) and reduce
//                          with shuffles.  The
//                          last warp to finish an item (shared-memory counter)
//                          merges the warps' results and writes the item's partial
//                          as self-validating tagged words (below).  Consumers
//                          never wait on global memory and issue no fences.
//   issuer (warp 16)       one lane fills stages with 1-D bulk copies
//                          (cp.async.bulk, no multicast) completing on the stage's
//                          "full" mbarrier.  It touches only shared memory.
//   scheduler (warp 17)    one lane claims items from a global counter, decodes
//                          them, resolves residual items once their sequence's
//                          outcome is known, and queues ready-to-issue items for the
//                          issuer in shared memory.
//   publisher (warp 18)    writes the items' merged results to global memory.
// The split keeps every warp that arrives on a pipeline barrier free of global
// memory accesses in flight: a release (an mbarrier arrive) has to wait for the
// issuing warp's outstanding global loads and stores, which would put a memory
// round trip on every item.
//   finisher (warp 19)     owns sequences b = blockIdx.x, blockIdx.x + gridDim.x, ...
//                          It waits until every pass-1 partial of a sequence
//                          carries this call's tag, runs sequence_tail (fp64
//                          combine, gather, log-space accept scan [FlashSpec,
//                          Metodologia 1]), raises the ready flag, waits for the
//                          residual sums and draws the extra token [Speculative
//                          Speculative Decoding, Metodologia 2].  This overlaps
//                          with streaming.
//
// Publication by tags.  Each call has a tag (2 * epoch + 1 with bit 31 set, the
// epoch kept in the workspace; words the general path leaves behind never have
// that form in their upper half unless a logit times log2(e)/T exceeds 2^23).  Partials and residual sums are 64-bit words (value | tag << 32)
// written with relaxed stores: a naturally aligned 64-bit access is single-copy
// atomic, so a reader that sees the current tag in a word also sees its value,
// and no release fence is needed on the hot path.  Ready flags hold the tag
// (release / acquire, once per sequence).  Nothing has to be reset between
// calls: the last CTA to exit only rewinds the claim counter and bumps the epoch.
//
// No wait can hang: every mbarrier, flag and tag wait gives up after kWaitLimitNs
// of %globaltimer, records an error word in the workspace and makes the CTA wind
// down.
#pragma once

#include "sv_common.cuh"
#include "sv_generic.cuh"

namespace sv {

constexpr int kStages = 6;                   // shared-memory stages; consumer group g owns g, g+2, g+4
constexpr int kMaxItemBytes = 32768;
constexpr int kMinItemBytes = 4096;
constexpr int kSW = 16;                      // consumer warps, in two groups taking alternate items
constexpr int kGW = kSW / 2;                 // warps per consumer group
constexpr int kGT = kGW * 32;                // threads per consumer group
constexpr int kST = kSW * 32;                // consumer threads
constexpr int kStreamThreads = kST + 128;    // + issuer, scheduler, publisher, finisher warps
constexpr int kIssuerWarp = kSW;
constexpr int kSchedWarp = kSW + 1;
constexpr int kPubWarp = kSW + 2;
constexpr int kFinisherWarp = kSW + 3;
constexpr int kSQ = 32;                      // scheduler -> issuer queue
constexpr int kOB = 64;                      // consumers -> publisher queue
constexpr int kSlots = 2 * kStages;          // merge slots: item k uses slot k % kSlots
constexpr int kDrawStage = 1024;             // residual sums staged in shared memory for the draw
constexpr int kDefer = 32;                   // residual items a producer may hold back
constexpr int kClaim = 4;                    // items per claim of the global counter
constexpr int kVPT = kMaxItemBytes / 16 / kGT;  // 16-byte vectors per group thread per stage (8)
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

enum : int { kItemP1 = 0, kItemP2 = 1, kItemEnd = 3 };
enum : unsigned { kErrEmptyWait = 1u, kErrFullWait = 2u, kErrReadyWait = 4u, kErrCountWait = 8u };

struct __align__(16) ItemDesc {
    int kind;
    int b;
    int r;       // P1: row within the sequence; P2: row n of target and draft
    int c;       // chunk index within the row
    int bytes;   // P1: bytes of the row segment; P2: bytes of each half
    int v0;      // first element of the segment
    int two;     // P2: 1 when the draft half follows the target half
    int greedy;  // P1: temperature 0 (first argmax instead of the normaliser)
    SeqRec rec;  // P2: the sequence's outcome; P1: rec.k_hi / rec.k_lo = log2(e)/T
};

// A decoded item, ready to issue.
struct __align__(16) SchedEntry {
    ItemDesc d;
    const void* src0;
    const void* src1;
    unsigned tx;
    int pad[3];
};

// A merged result to publish: n words (value bits; the publisher adds the tag).
struct __align__(16) OutEntry {
    unsigned long long* dst;
    int n;
    int gen;  // (entry index / kOB) + 1 once filled
    unsigned w[kGW];
};

struct StreamCtl {
    unsigned tag;               // this call's publication tag
    SchedEntry sq[kSQ];
    int sq_tail;                // entries pushed by the scheduler
    int sq_head;                // entries taken by the issuer
    OutEntry ob[kOB];
    int ob_reserve;             // entries claimed by consumers
    int ob_head;                // entries published
    int cons_done;              // consumer warps that have finished
    unsigned long long full[kStages];
    unsigned long long empty[kStages];
    ItemDesc desc[kStages];
    float4 slot[kSlots][kGW];   // per-warp results of an item, merged by its last warp
    double dslot[kSlots][kGW];
    int done[kSlots];           // warp results written into the slot, over all its uses
    int merged[kSlots];         // merges finished on the slot, over all its uses
    long long issued;           // stages handed to the consumers (issuer)
    long long consumed;         // stages taken by the consumers
    int abort;
};

struct StreamArgs {
    TailArgs t;                    // t.nc = nI1 partials per row
    unsigned long long* pw;        // [B][R][nI1][2] tagged partial words
    const float* u_resample;
    unsigned* ready;               // [B] the tag once the sequence's outcome is known
    unsigned long long* counters;  // [0] next item, [1] CTAs finished, [2] error bits, [3] epoch
    unsigned long long* rw;        // [B][nI2][kGW] tagged residual sums per (item, warp range)
    int IB;                        // stage bytes; P1 segment <= IB, P2 half <= IB/2
    int nI1, nI2, D, per_step;
    long long n_items;
    long long rowbytes;
};

// ----------------------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p);

__device__ __forceinline__ int ld_acquire_shared(const int* p)
{
    int v;
    asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_shared(int* p, int v)
{
    asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(unsigned long long* bar, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(unsigned long long* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_tx(unsigned long long* bar, unsigned bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// non-blocking test of a phase
__device__ __forceinline__ bool mbar_test_wait(unsigned long long* bar, unsigned parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Blocking test of a phase: the thread sleeps until the phase completes or a
// time-limit hint (ns) expires, so a waiting warp does not take issue slots.
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, unsigned parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase with the given parity; false after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(unsigned long long* bar, unsigned parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (unsigned it = 1; it < (1u << 30); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
    return false;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, unsigned long long* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned* p)
{
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_acquire_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

__device__ __forceinline__ void st_release(unsigned* p, unsigned v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// add without returning: the issuing thread does not wait for it
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Spin (with back-off) until *p == want; false after kWaitLimitNs.
__device__ __forceinline__ bool wait_equal(const unsigned* p, unsigned want)
{
    if (ld_acquire(p) == want) return true;
    const unsigned long long t0 = global_ns();
    for (unsigned it = 0; it < (1u << 30); ++it) {
        __nanosleep(64);
        if (ld_acquire(p) == want) return true;
        if ((it & 15u) == 0 && global_ns() - t0 > kWaitLimitNs) return false;
    }
    return false;
}

// One warp waits until every word of p[0, n) carries `tag` in its upper half;
// false after kWaitLimitNs.  Each pass reads up to 256 words per round trip
// (8 independent loads per lane) and restarts from the first stale word.
__device__ __forceinline__ bool wait_tagged(const unsigned long long* p, int n, unsigned tag)
{
    const int lane = threadIdx.x & 31;
    const unsigned long long t0 = global_ns();
    int from = 0;  // every word below `from` has been seen tagged
    for (;;) {
        int bad = n;
        for (int base = from; base < n; base += 256) {
            unsigned long long v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int idx = base + j * 32 + lane;
                v[j] = idx < n ? ld_relaxed_u64(p + idx) : ((unsigned long long)tag << 32);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if ((unsigned)(v[j] >> 32) != tag) bad = min(bad, base + j * 32 + lane);
            if (__any_sync(0xffffffffu, bad < n)) break;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bad = min(bad, __shfl_xor_sync(0xffffffffu, bad, o));
        if (bad >= n) return true;
        from = bad;
        if (global_ns() - t0 > kWaitLimitNs) return false;
        __nanosleep(64);
    }
}

// SeqRec written by another CTA: read it at L2 (after the acquire on its ready flag)
__device__ __forceinline__ SeqRec load_seqrec_cg(const SeqRec* p)
{
    union {
        int4 v[2];
        SeqRec r;
    } u;
    u.v[0] = __ldcg(reinterpret_cast<const int4*>(p));
    u.v[1] = __ldcg(reinterpret_cast<const int4*>(p) + 1);
    return u.r;
}

__device__ __forceinline__ void record_error(const StreamArgs& a, StreamCtl& ctl, unsigned bits)
{
    atomicOr(&a.counters[2], (unsigned long long)bits);
    *(volatile int*)&ctl.abort = 1;
}

template <int ESZ>
__device__ __forceinline__ const unsigned char* row_ptr(const TailArgs& t, int b, int r)
{
    const size_t V = (size_t)t.V;
    return r <= t.gamma
               ? static_cast<const unsigned char*>(t.tgt) + ((size_t)b * (t.gamma + 1) + r) * V * ESZ
               : static_cast<const unsigned char*>(t.dft) + ((size_t)b * t.gamma + (r - t.gamma - 1)) * V * ESZ;
}

// Item k goes to consumer group k % 2, which owns stages g, g+2, g+4 and takes
// its items in order; so each stage is filled and drained by one group only and
// a waiter is never more than one phase ahead of its barrier.
__device__ __forceinline__ int stage_of(long long k) { return 2 * (int)((k >> 1) % 3) + (int)(k & 1); }
__device__ __forceinline__ unsigned phase_of(long long k) { return (unsigned)(((k >> 1) / 3) & 1); }

// ----------------------------------------------------------------------------- producer

// Scheduler.  Items are claimed kClaim at a time.  A residual item of sequence b
// can only be issued once b's outcome is known.  Instead of blocking on b's ready
// flag, the scheduler parks such an item (up to kDefer of them) and keeps going;
// parked items are retried first (every fourth push at most, since each check is
// a memory round trip) and drained, blocking, once the claims run out.  Every
// parked item depends only on work claimed before it, so this cannot deadlock.
// All of its global loads complete before it pushes (a release) to the queue.
template <int ESZ>
__device__ void stream_scheduler(const StreamArgs& a, StreamCtl& ctl)
{
    __shared__ int2 s_defer[kDefer];  // (b, c) of parked residual items, oldest first
    const TailArgs& t = a.t;
    const int B = (int)(a.n_items / a.per_step) - a.D;
    const int P1 = t.R * a.nI1;
    const int half = a.IB / 2;
    const unsigned tag = ctl.tag;
    const unsigned n_items = (unsigned)a.n_items;
    const unsigned per_step = (unsigned)a.per_step;
    int pushed = 0;
    bool ok = true;
    int last_b = -1, ndef = 0, since_peek = 0;
    float T_last = 0.f, khi = 0.f, klo = 0.f;
    bool claims_left = true;
    int rec_b = -1;  // sequence whose outcome is cached in rec_c
    SeqRec rec_c;
    unsigned i = 0, i_end = 0;

    auto push = [&](const SchedEntry& e) -> bool {
        if (pushed - *(volatile int*)&ctl.sq_head >= kSQ) {
            const unsigned long long t0 = global_ns();
            while (pushed - *(volatile int*)&ctl.sq_head >= kSQ) {
                if (*(volatile int*)&ctl.abort) return false;
                if (global_ns() - t0 > kWaitLimitNs) { record_error(a, ctl, kErrEmptyWait); return false; }
                __nanosleep(32);
            }
        }
        ctl.sq[pushed % kSQ] = e;
        st_release_shared(&ctl.sq_tail, pushed + 1);
        ++pushed;
        return true;
    };

    for (;;) {
        if (*(volatile int*)&ctl.abort) { ok = false; break; }
        SchedEntry e;
        ItemDesc& d = e.d;
        d.greedy = 0;
        d.two = 0;
        e.tx = 0;
        e.src0 = nullptr;
        e.src1 = nullptr;
        int p2_b = -1, p2_c = 0;

        // 1) a parked residual item whose sequence is ready now (or must be drained)
        if (ndef > 0) {
            const bool drain = !claims_left || ndef == kDefer;
            const int2 o = s_defer[0];
            bool ready = o.x == rec_b;
            if (!ready && (drain || ++since_peek >= 4)) {
                since_peek = 0;
                ready = ld_relaxed_u32(&a.ready[o.x]) == tag;
                if (!ready && drain) {
                    if (!wait_equal(&a.ready[o.x], tag)) { record_error(a, ctl, kErrReadyWait); ok = false; break; }
                    ready = true;
                }
            }
            if (ready) {
                p2_b = o.x;
                p2_c = o.y;
                for (int j = 1; j < ndef; ++j) s_defer[j - 1] = s_defer[j];
                --ndef;
            }
        }
        // 2) otherwise the next claimed item
        if (p2_b < 0) {
            if (!claims_left) {
                if (ndef == 0) break;
                continue;
            }
            if (i >= i_end) {
                i = (unsigned)atomicAdd(&a.counters[0], (unsigned long long)kClaim);
                i_end = i + kClaim;
            }
            if (i >= n_items) {
                claims_left = false;
                continue;
            }
            const unsigned cur = i++;
            const unsigned ss = cur / per_step;
            const int kk = (int)(cur - ss * per_step);
            if (kk < P1) {
                if (ss >= (unsigned)B) continue;
                const int b = (int)ss, r = kk / a.nI1, c = kk - (kk / a.nI1) * a.nI1;
                if (b != last_b) {
                    T_last = t.temperature[b];
                    if (T_last != 0.f && temperature_ok(T_last)) split_k(T_last, &khi, &klo);
                    last_b = b;
                }
                const float T = T_last;
                if (!(temperature_ok(T) && !(T == 0.f && r > t.gamma))) continue;  // never read
                const long long off = (long long)c * a.IB;
                const long long left = a.rowbytes - off;
                d.kind = kItemP1;
                d.b = b;
                d.r = r;
                d.c = c;
                d.bytes = (int)(left < a.IB ? left : a.IB);
                d.v0 = (int)(off / ESZ);
                d.greedy = (T == 0.f);
                d.rec.k_hi = khi;
                d.rec.k_lo = klo;
                e.src0 = row_ptr<ESZ>(t, b, r) + off;
                e.tx = (unsigned)d.bytes;
            } else {
                const int bb = (int)ss - a.D;
                if (bb < 0 || bb >= B) continue;
                const int b = bb, c = kk - P1;
                if (b != rec_b && ld_relaxed_u32(&a.ready[b]) != tag) {  // not known yet: park it
                    s_defer[ndef++] = make_int2(b, c);
                    continue;
                }
                p2_b = b;
                p2_c = c;
            }
        }
        if (p2_b >= 0) {
            if (p2_b != rec_b) {  // the ready flag was seen: acquire, then its outcome
                fence_acquire_gpu();
                rec_c = load_seqrec_cg(t.seq + p2_b);
                rec_b = p2_b;
            }
            const SeqRec rec = rec_c;
            if (rec.mode == kModeNone) continue;
            const long long off = (long long)p2_c * half;
            const long long left = a.rowbytes - off;
            d.kind = kItemP2;
            d.b = p2_b;
            d.r = rec.n;
            d.c = p2_c;
            d.bytes = (int)(left < half ? left : half);
            d.v0 = (int)(off / ESZ);
            d.two = rec.mode == kModeResidual;
            d.rec = rec;
            e.src0 = row_ptr<ESZ>(t, p2_b, rec.n) + off;
            if (d.two) e.src1 = row_ptr<ESZ>(t, p2_b, t.gamma + 1 + rec.n) + off;
            e.tx = (unsigned)d.bytes * (d.two ? 2u : 1u);
        }
        if (!push(e)) { ok = false; break; }
    }
    for (int k = 0; ok && k < 2; ++k) {  // one end marker per consumer group
        SchedEntry e;
        e.d.kind = kItemEnd;
        e.tx = 0;
        e.src0 = e.src1 = nullptr;
        if (!push(e)) break;
    }
}

// Issuer: takes the scheduler's entries in order and fills the stages.  Only
// shared memory, mbarriers and bulk-copy issue happen here.
__device__ void stream_issuer(const StreamArgs& a, StreamCtl& ctl, unsigned char* stages)
{
    const int half = a.IB / 2;
    long long k = 0;
    int ends = 0;
    while (ends < 2) {
        if (ld_acquire_shared(&ctl.sq_tail) <= (int)k) {
            const unsigned long long t0 = global_ns();
            bool got = false;
            for (;;) {
                if (ld_acquire_shared(&ctl.sq_tail) > (int)k) { got = true; break; }
                if (*(volatile int*)&ctl.abort) break;
                if (global_ns() - t0 > kWaitLimitNs) { record_error(a, ctl, kErrEmptyWait); break; }
                __nanosleep(20);
            }
            if (!got) break;
        }
        const SchedEntry e = ctl.sq[k % kSQ];
        st_release_shared(&ctl.sq_head, (int)k + 1);
        const int s = stage_of(k);
        if (!mbar_wait(&ctl.empty[s], phase_of(k) ^ 1u)) { record_error(a, ctl, kErrEmptyWait); break; }
        ctl.desc[s] = e.d;
        if (e.d.kind == kItemEnd) {
            mbar_arrive(&ctl.full[s]);
            ++ends;
        } else {
            mbar_arrive_tx(&ctl.full[s], e.tx);
            bulk_g2s(stages + (size_t)s * a.IB, e.src0, (unsigned)e.d.bytes, &ctl.full[s]);
            if (e.src1) bulk_g2s(stages + (size_t)s * a.IB + half, e.src1, (unsigned)e.d.bytes, &ctl.full[s]);
        }
        ++k;
    }
    ctl.issued = k;
}

// Publisher: writes each merged result as tagged words, in the order the
// consumers queued them, until every consumer warp has finished.
__device__ void stream_publisher(const StreamArgs& a, StreamCtl& ctl)
{
    const int lane = threadIdx.x & 31;
    const unsigned long long tagw = (unsigned long long)ctl.tag << 32;
    long long h = 0;
    unsigned long long t0 = global_ns();
    for (;;) {
        OutEntry& e = ctl.ob[h % kOB];
        const int want = (int)(h / kOB) + 1;
        if (ld_acquire_shared(&e.gen) == want) {
            const int n = e.n;
            unsigned long long* dst = e.dst;
            // the stores depend on the entry's values, so once they are issued the
            // entry has been read and may be reused (no release needed here)
            if (lane < n) st_relaxed_u64(dst + lane, tagw | e.w[lane]);
            __syncwarp();
            if (lane == 0) *(volatile int*)&ctl.ob_head = (int)h + 1;
            ++h;
            t0 = global_ns();
            continue;
        }
        int fin = 0;
        if (lane == 0)
            fin = (*(volatile int*)&ctl.cons_done == kSW) && (*(volatile int*)&ctl.ob_reserve == (int)h);
        if (__shfl_sync(0xffffffffu, fin, 0)) break;
        if (global_ns() - t0 > kWaitLimitNs) {
            if (lane == 0) record_error(a, ctl, kErrCountWait);
            break;
        }
        __nanosleep(32);
    }
}

// Lane 0 of a consumer warp queues a merged result for the publisher.
__device__ __forceinline__ void queue_result(const StreamArgs& a, StreamCtl& ctl, unsigned long long* dst, int n,
                                             const unsigned* w)
{
    const int idx = atomicAdd(&ctl.ob_reserve, 1);
    if (idx - *(volatile int*)&ctl.ob_head >= kOB) {
        const unsigned long long t0 = global_ns();
        while (idx - *(volatile int*)&ctl.ob_head >= kOB) {
            if (global_ns() - t0 > kWaitLimitNs) { record_error(a, ctl, kErrFullWait); return; }
            __nanosleep(32);
        }
    }
    OutEntry& e = ctl.ob[idx % kOB];
    e.dst = dst;
    e.n = n;
    for (int i = 0; i < n; ++i) e.w[i] = w[i];
    st_release_shared(&e.gen, idx / kOB + 1);
}

// ----------------------------------------------------------------------------- consumers

// Lane 0 of a warp takes its turn on a merge slot: wait (bounded) until the
// slot's previous use has been merged, which is normally already the case.
__device__ __forceinline__ void slot_arrive(StreamCtl& ctl, int slot, int use)
{
    if (*(volatile int*)&ctl.merged[slot] < use) {
        const unsigned long long t0 = global_ns();
        while (*(volatile int*)&ctl.merged[slot] < use && global_ns() - t0 < kWaitLimitNs) __nanosleep(32);
    }
}

template <int ESZ>
__device__ void stream_consumer_warp(const StreamArgs& a, StreamCtl& ctl, const unsigned char* stages, int grp)
{
    constexpr int VEC = 16 / ESZ;
    const TailArgs& t = a.t;
    const int lane = threadIdx.x & 31;
    const int gw = (threadIdx.x >> 5) - grp * kGW;  // warp within the group
    const int gtid = gw * 32 + lane;                // thread within the group
    const int half = a.IB / 2;
    const uint4 kNegInf = ESZ == 2 ? make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u)
                                   : make_uint4(0xff800000u, 0xff800000u, 0xff800000u, 0xff800000u);
    for (long long k = grp;; k += 2) {
        const int s = stage_of(k);
        const int slot = (int)(k % kSlots);
        const int use = (int)(k / kSlots);
        const unsigned par = phase_of(k);
        // lane 0 does the bounded wait; the warp follows its decision, then every
        // lane observes the completed phase itself (acquire for its own reads)
        int ok = 0;
        if (lane == 0) ok = mbar_wait(&ctl.full[s], par) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
            if (lane == 0) record_error(a, ctl, kErrFullWait);
            break;
        }
        (void)mbar_test_wait(&ctl.full[s], par);  // completed: acquire for this lane
        const ItemDesc d = ctl.desc[s];
        if (lane == 0) atomicMax(reinterpret_cast<unsigned long long*>(&ctl.consumed), (unsigned long long)(k + 1));
        if (d.kind == kItemEnd) break;
        const unsigned char* st = stages + (size_t)s * a.IB;

        if (d.kind == kItemP1) {
            const uint4* sp = reinterpret_cast<const uint4*>(st);
            const int nvec = d.bytes >> 4;
            float4 res;
            if (!d.greedy) {
                const float khi = d.rec.k_hi, klo = d.rec.k_lo;
                // this thread's vectors in registers; one offset for the whole warp
                // (its largest logit), then every exponent against it
                uint4 v[kVPT];
#pragma unroll
                for (int j = 0; j < kVPT; ++j) {
                    const int i = gtid + j * kGT;
                    v[j] = i < nvec ? sp[i] : kNegInf;
                }
                float m = vec_max<ESZ>(v[0]);
#pragma unroll
                for (int j = 1; j < kVPT; ++j) m = fmaxf(m, vec_max<ESZ>(v[j]));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                const float mk = (m == -INFINITY) ? 0.f : ceilf(__fmul_rn(m, khi));
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < kVPT; ++j) {
                    float x[VEC];
                    unpack<ESZ>(v[j], x);
#pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[(j * VEC + e) & 7] += scaled_exp(x[e], khi, klo, mk);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.empty[s]);
                float sum = tree8(acc);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                res = make_float4(m, mk, m == -INFINITY ? 0.f : sum, 0.f);
            } else {
                Amax A{-INFINITY, 0x7fffffff, 0};
                for (int i = gtid; i < nvec; i += kGT) {
                    float x[VEC];
                    unpack<ESZ>(sp[i], x);
#pragma unroll
                    for (int e = 0; e < VEC; ++e) amax_add(A, x[e], d.v0 + i * VEC + e);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.empty[s]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ob = __shfl_xor_sync(0xffffffffu, A.best, o);
                    const int oi = __shfl_xor_sync(0xffffffffu, A.idx, o);
                    const int on = __shfl_xor_sync(0xffffffffu, A.nan, o);
                    amax_merge(A, ob, oi, on);
                }
                res = make_float4(A.best, 0.f, (float)A.nan, __int_as_float(A.idx));
            }
            // hand the warp's result to the item's last warp in this group
            int last = 0;
            if (lane == 0) {
                slot_arrive(ctl, slot, use);
                ctl.slot[slot][gw] = res;
                __threadfence_block();
                last = (atomicAdd(&ctl.done[slot], 1) == (use + 1) * kGW - 1);
            }
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                __threadfence_block();
                const float4 q = lane < kGW ? ctl.slot[slot][lane] : make_float4(-INFINITY, 0.f, 0.f, 0.f);
                __syncwarp();
                if (lane == 0) {
                    __threadfence_block();
                    ctl.merged[slot] = use + 1;  // the slot may be reused
                }
                Partial p;
                if (!d.greedy) {
                    Lse L{q.x, q.y, q.z};
                    if (lane >= kGW) lse_init(L);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        const float om = __shfl_xor_sync(0xffffffffu, L.m, o);
                        const float omk = __shfl_xor_sync(0xffffffffu, L.mk, o);
                        const float os = __shfl_xor_sync(0xffffffffu, L.s, o);
                        lse_merge(L, om, omk, os);
                    }
                    p = Partial{L.m, L.mk, L.s, 0};
                } else {
                    Amax A{q.x, lane < kGW ? __float_as_int(q.w) : 0x7fffffff, lane < kGW ? (q.z != 0.f) : 0};
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        const float ob = __shfl_xor_sync(0xffffffffu, A.best, o);
                        const int oi = __shfl_xor_sync(0xffffffffu, A.idx, o);
                        const int on = __shfl_xor_sync(0xffffffffu, A.nan, o);
                        amax_merge(A, ob, oi, on);
                    }
                    p = Partial{A.best, 0.f, (float)A.nan, A.idx};
                }
                if (lane == 0) {
                    const unsigned w[2] = {__float_as_uint(p.m),
                                           d.greedy ? ((unsigned)p.idx | ((p.s != 0.f) ? 0x80000000u : 0u))
                                                    : __float_as_uint(p.s)};
                    queue_result(a, ctl, a.pw + 2 * (((size_t)d.b * t.R + d.r) * a.nI1 + d.c), 2, w);
                }
            }
        } else {  // kItemP2: this warp sums a contiguous range of the item
            const uint4* tp = reinterpret_cast<const uint4*>(st);
            const uint4* dp = reinterpret_cast<const uint4*>(st + half);
            const int nvec = d.bytes >> 4;
            const int Q = (nvec + kGW - 1) / kGW;
            const int q0 = gw * Q, q1 = min(nvec, q0 + Q);
            const bool p_only = !d.two;
            constexpr int kH = kVPT / 2;
            double acc0 = 0.0, acc1 = 0.0;
            for (int g0 = q0 + lane; g0 < q1; g0 += kH * 32) {
                uint4 vt[kH], vd[kH];
#pragma unroll
                for (int j = 0; j < kH; ++j) {
                    const int q = g0 + j * 32;
                    vt[j] = q < q1 ? tp[q] : kNegInf;
                    vd[j] = (q < q1 && !p_only) ? dp[q] : kNegInf;
                }
#pragma unroll
                for (int j = 0; j < kH; ++j) {
                    float xt[VEC], xd[VEC], w[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    unpack<ESZ>(vt[j], xt);
                    unpack<ESZ>(vd[j], xd);
#pragma unroll
                    for (int e = 0; e < VEC; ++e) w[e] = weight_of(d.rec, p_only, xt[e], p_only ? 0.f : xd[e]);
                    if (j & 1) acc1 += (double)tree8(w);
                    else acc0 += (double)tree8(w);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.empty[s]);
            const double acc = warp_sum(acc0 + acc1);
            int last = 0;
            if (lane == 0) {
                slot_arrive(ctl, slot, use);
                ctl.dslot[slot][gw] = acc;
                __threadfence_block();
                last = (atomicAdd(&ctl.done[slot], 1) == (use + 1) * kGW - 1);
            }
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last && lane == 0) {
                __threadfence_block();
                unsigned w[kGW];
#pragma unroll
                for (int j = 0; j < kGW; ++j) w[j] = __float_as_uint((float)ctl.dslot[slot][j]);
                __threadfence_block();
                ctl.merged[slot] = use + 1;
                queue_result(a, ctl, a.rw + ((size_t)d.b * a.nI2 + d.c) * kGW, kGW, w);
            }
        }
    }
    __syncwarp();
    if (lane == 0) atomicAdd(&ctl.cons_done, 1);
}

// ----------------------------------------------------------------------------- draw

// Scan uint4 indices [q0, q1) of the row pair in order with one warp.  Up to
// kPre groups of 32 vectors are loaded before any of them is used, so a range of
// kPre*32 vectors costs one memory latency.  Returns the first element whose
// running sum (from `base`) exceeds `target`, or -1; *lastpos gets the last
// element in the range with a positive weight, *total the range's weight sum.
template <int ESZ>
__device__ long long warp_scan_range(const unsigned char* trow, const unsigned char* drow, const SeqRec& rec,
                                     bool p_only, long long q0, long long q1, double base, double target,
                                     long long* lastpos, double* total)
{
    constexpr int VEC = 16 / ESZ;
    constexpr int kPre = 4;
    const int lane = threadIdx.x & 31;
    const uint4* tv = reinterpret_cast<const uint4*>(trow);
    const uint4* dv = reinterpret_cast<const uint4*>(drow);
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    double run = base;
    long long last = -1, hit = -1;
    for (long long g0 = q0; g0 < q1 && hit < 0; g0 += 32 * kPre) {
        uint4 vt[kPre], vd[kPre];
#pragma unroll
        for (int j = 0; j < kPre; ++j) {
            const long long q = g0 + j * 32 + lane;
            vt[j] = q < q1 ? __ldcg(tv + q) : zero;
            vd[j] = (q < q1 && !p_only) ? __ldcg(dv + q) : zero;
        }
#pragma unroll
        for (int j = 0; j < kPre; ++j) {
            const long long q = g0 + j * 32 + lane;
            if (g0 + j * 32 >= q1) break;
            float w[VEC];
            double loc = 0.0;
            float xt[VEC], xd[VEC];
            unpack<ESZ>(vt[j], xt);
            unpack<ESZ>(vd[j], xd);
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                w[e] = q < q1 ? weight_of(rec, p_only, xt[e], p_only ? 0.f : xd[e]) : 0.f;
                loc += (double)w[e];
            }
            const double incl = warp_inclusive_scan(loc);
            double c = run + incl - loc;
            long long my_hit = -1, my_last = -1;
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                c += (double)w[e];
                if (my_hit < 0 && w[e] > 0.f && c > target) my_hit = q * VEC + e;
                if (w[e] > 0.f) my_last = q * VEC + e;
            }
            const unsigned hm = __ballot_sync(0xffffffffu, my_hit >= 0);
            const unsigned lm = __ballot_sync(0xffffffffu, my_last >= 0);
            if (lm) last = __shfl_sync(0xffffffffu, my_last, 31 - __clz(lm));
            run += __shfl_sync(0xffffffffu, incl, 31);
            if (hm) {
                hit = __shfl_sync(0xffffffffu, my_hit, __ffs(hm) - 1);
                break;
            }
        }
    }
    *lastpos = last;
    *total = run - base;
    return hit;
}

// Inverse CDF for sequence b from the per-(item, warp) residual sums, on one
// warp: the item holding u*S, then the warp range inside it, then the token.
template <int ESZ>
__device__ void stream_draw(const StreamArgs& a, int b, const SeqRec& rec)
{
    __shared__ double s_rs[kDrawStage];
    const int lane = threadIdx.x & 31;
    const TailArgs& t = a.t;
    const int nI2 = a.nI2;
    const long long half = a.IB / 2;
    const unsigned long long* rs_g = a.rw + (size_t)b * nI2 * kGW;
    const int nrs = nI2 * kGW;
    const bool staged = nrs <= kDrawStage;
    if (staged) {
        for (int i0 = 0; i0 < nrs; i0 += 256) {  // 8 independent loads per lane per round trip
            unsigned long long v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = (i0 + j * 32 + lane < nrs) ? ld_relaxed_u64(rs_g + i0 + j * 32 + lane) : 0ull;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (i0 + j * 32 + lane < nrs) s_rs[i0 + j * 32 + lane] = (double)__uint_as_float((unsigned)v[j]);
        }
        __syncwarp();
    }
    auto rsv = [&](int i) {
        return staged ? s_rs[i] : (double)__uint_as_float((unsigned)ld_relaxed_u64(rs_g + i));
    };
    auto item_sum = [&](int c) {
        double s = 0.0;
        for (int w = 0; w < kGW; ++w) s += rsv(c * kGW + w);
        return s;
    };
    const unsigned char* trow = row_ptr<ESZ>(t, b, rec.n);
    const unsigned char* drow = rec.mode == kModeResidual ? row_ptr<ESZ>(t, b, t.gamma + 1 + rec.n) : nullptr;
    const bool bonus = rec.mode == kModeBonus;
    const long long nq_row = a.rowbytes / 16;
    const double u = (double)a.u_resample[b];

    double S = 0.0;
    for (int c0 = 0; c0 < nI2; c0 += 32) {
        const int c = c0 + lane;
        S += __shfl_sync(0xffffffffu, warp_inclusive_scan(c < nI2 ? item_sum(c) : 0.0), 31);
    }

    long long token = -1;
    int flag = 0;
    if (!(S > 0.0) && !bonus) {
        // the residual vanished (p == q up to rounding): draw from p_n over the whole row
        flag = SV_ROW_RESIDUAL_ZERO;
        long long lp;
        double Sp;
        warp_scan_range<ESZ>(trow, nullptr, rec, true, 0, nq_row, 0.0, INFINITY, &lp, &Sp);
        double tot;
        token = warp_scan_range<ESZ>(trow, nullptr, rec, true, 0, nq_row, 0.0, u * Sp, &lp, &tot);
        if (token < 0) token = lp;
    } else {
        const double target = u * S;
        // item c*: first item whose inclusive prefix exceeds the target
        double carry = 0.0, base = 0.0;
        int cstar = -1, clast = -1;
        for (int c0 = 0; c0 < nI2 && cstar < 0; c0 += 32) {
            const int c = c0 + lane;
            const double v = c < nI2 ? item_sum(c) : 0.0;
            const double incl = carry + warp_inclusive_scan(v);
            const unsigned hm = __ballot_sync(0xffffffffu, c < nI2 && incl > target);
            const unsigned pm = __ballot_sync(0xffffffffu, c < nI2 && v > 0.0);
            if (pm) clast = c0 + 31 - __clz(pm);
            if (hm) {
                const int l = __ffs(hm) - 1;
                cstar = c0 + l;
                base = __shfl_sync(0xffffffffu, incl - v, l);
            }
            carry = __shfl_sync(0xffffffffu, incl, 31);
        }
        const bool take_last = cstar < 0;
        if (take_last) cstar = clast;
        if (cstar >= 0) {
            // warp range w* inside item c*
            int wstar = -1, wlast = -1;
            double run = base;
            for (int w = 0; w < kGW; ++w) {
                const double v = rsv(cstar * kGW + w);
                if (v > 0.0) wlast = w;
                if (!take_last && wstar < 0 && run + v > target) { wstar = w; break; }
                run += v;
            }
            const bool last_sub = wstar < 0;
            if (last_sub) {
                wstar = wlast;
                run = base;
                for (int w = 0; w < wstar; ++w) run += rsv(cstar * kGW + w);
            }
            if (wstar >= 0) {
                const long long left = a.rowbytes - (long long)cstar * half;
                const int nvec = (int)((left < half ? left : half) >> 4);
                const int Q = (nvec + kGW - 1) / kGW;
                const long long q0 = (long long)cstar * (half >> 4) + (long long)wstar * Q;
                const long long q1 = (long long)cstar * (half >> 4) + (long long)min(nvec, (wstar + 1) * Q);
                long long lp;
                double tot;
                token = warp_scan_range<ESZ>(trow, drow, rec, bonus, q0, q1, run,
                                             (take_last || last_sub) ? INFINITY : target, &lp, &tot);
                if (token < 0) token = lp;
            }
        }
    }
    if (lane == 0) {
        t.out_tokens[(size_t)b * (t.gamma + 1) + rec.n] = (int)token;
        if (flag && t.out_status) t.out_status[b] |= flag;
    }
    __syncwarp();
}

// ----------------------------------------------------------------------------- finisher

template <int ESZ>
__device__ void stream_finisher(const StreamArgs& a, StreamCtl& ctl)
{
    const int lane = threadIdx.x & 31;
    const TailArgs& t = a.t;
    const int B = (int)(a.n_items / a.per_step) - a.D;
    const unsigned tag = ctl.tag;
    for (int b = blockIdx.x; b < B; b += gridDim.x) {
        const float T = t.temperature[b];
        const int rows = !temperature_ok(T) ? 0 : (T == 0.f ? t.gamma + 1 : t.R);
        int ok = wait_tagged(a.pw + 2 * (size_t)b * t.R * a.nI1, 2 * rows * a.nI1, tag) ? 1 : 0;
        if (!ok) {
            if (lane == 0) record_error(a, ctl, kErrCountWait);
            return;
        }
        sequence_tail<ESZ, 32, WarpSync>(t, b, lane, TaggedPartials{a.pw});
        __syncwarp();
        if (lane == 0) {
            __threadfence();
            st_release(&a.ready[b], tag);
        }
        const SeqRec rec = t.seq[b];  // written by this warp's lane 0 above
        if (rec.mode == kModeNone) continue;
        ok = wait_tagged(a.rw + (size_t)b * a.nI2 * kGW, a.nI2 * kGW, tag) ? 1 : 0;
        if (!ok) {
            if (lane == 0) record_error(a, ctl, kErrCountWait);
            return;
        }
        stream_draw<ESZ>(a, b, rec);
    }
}

// ----------------------------------------------------------------------------- kernel

template <int ESZ>
__global__ void __launch_bounds__(kStreamThreads, 1) sv_stream(StreamArgs a)
{
    extern __shared__ __align__(128) unsigned char sv_stage_mem[];
    __shared__ StreamCtl ctl;
    __shared__ int s_exit_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctl.full[s], 1);
            mbar_init(&ctl.empty[s], kGW);
        }
        for (int s = 0; s < kSlots; ++s) ctl.done[s] = ctl.merged[s] = 0;
        for (int i = 0; i < kOB; ++i) ctl.ob[i].gen = 0;
        ctl.sq_tail = ctl.sq_head = 0;
        ctl.ob_reserve = ctl.ob_head = 0;
        ctl.cons_done = 0;
        ctl.tag = 0x80000000u | (2u * (unsigned)ld_relaxed_u64(&a.counters[3]) + 1u);
        ctl.abort = 0;
        ctl.issued = 0;
        ctl.consumed = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == kIssuerWarp) {
        if (lane == 0) stream_issuer(a, ctl, sv_stage_mem);
    } else if (warp == kSchedWarp) {
        if (lane == 0) stream_scheduler<ESZ>(a, ctl);
    } else if (warp == kPubWarp) {
        stream_publisher(a, ctl);
    } else if (warp == kFinisherWarp) {
        stream_finisher<ESZ>(a, ctl);
    } else {
        stream_consumer_warp<ESZ>(a, ctl, sv_stage_mem, warp / kGW);
    }
    __syncthreads();

    // copies still in flight (only after an error): at most the last kStages issued
    // stages can be outstanding, since a stage is refilled only after its previous
    // copy was waited for; let them land before the CTA exits
    if (threadIdx.x == 0) {
        for (long long k = ctl.issued > kStages ? ctl.issued - kStages : 0; k < ctl.issued; ++k)
            mbar_wait(&ctl.full[stage_of(k)], phase_of(k));
        __threadfence();
        const unsigned long long prev = atomicAdd(&a.counters[1], 1ull);
        s_exit_last = (prev == (unsigned long long)gridDim.x - 1ull);
    }
    __syncthreads();
    if (s_exit_last && threadIdx.x == 0) {
        // every other CTA has finished: rewind the claim counter, next call's tag
        __threadfence();
        a.counters[0] = 0ull;
        a.counters[1] = 0ull;
        a.counters[3] = a.counters[3] + 1ull;
    }
}

}  // namespace sv
