// spec_verify.cu -- C ABI of the B200 batched speculative-sampling verifier.
// The operation is specified in include/spec_verify.h.  This file plans a call
// (which kernel family, how the vocabulary is split, where everything lives in
// the workspace) and launches it:
//   * sv_stream + sv_draw (sv_pass.cuh): a persistent streaming kernel that
//     reads every logit once, then a programmatic dependent that finishes each
//     sequence, sums its draw rows (mostly from L2) and draws.  Used when every
//     row is 16-byte aligned (V * element size a multiple of 16) and at least
//     4 KB long.  Every slot these kernels read, the same call wrote.
//   * sv_small (sv_small.cuh): rows of at most kSmallMaxV elements; a group of
//     8, 16 or 32 lanes per sequence with the rows in registers, one launch, no
//     workspace traffic.
//   * sv_reset + sv_rowpass + sv_resample (sv_generic.cuh): any other shape;
//     sv_reset zeroes the per-sequence tickets first, so a workspace carries
//     nothing from one call to the next.
// SPEC_VERIFY_FORCE_GENERIC=1 in the environment selects the generic family for
// every shape (both compute the same results; tests use it to cover both).
#include "spec_verify.h"

#include <cuda.h>  // CUcontext / CUresult types only: driver calls go through entry points
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <algorithm>
#include <mutex>
#include <cstring>

#include "sv_common.cuh"
#include "sv_generic.cuh"
#include "sv_pass.cuh"
#include "sv_small.cuh"
#include "sv_topf.cuh"
#include "sv_bandit.cuh"
#include "sv_tree.cuh"
#include "sv_lowrank.cuh"

namespace {

using namespace sv;

constexpr int kSmCount = 148;             // B200; used only to size the split of V
constexpr int kPass1ChunkBytes = 32768;   // generic: bytes of one row streamed by one CTA
constexpr int kPass1MinChunk = 1024;      // generic: elements
constexpr int kPass2Chunk = 8192;         // generic: elements per residual CTA
constexpr int kPass2MinChunk = 512;
constexpr int kMaxDevices = 64;
// streaming path: the last rows streamed that are meant to stay in L2 for the
// draw (the rest load with an evict-first hint); about 2/3 of the 126 MB L2
constexpr long long kL2KeepBytes = 80LL << 20;

struct Plan {
    int B, gamma, V, R, esz;
    bool small, stream;
    int nc1, C1, nc2, C2;           // generic
    int nslot, NT2;                 // stream
    long long evict_rows;           // stream: rows loaded evict-first
    long long nq;                   // stream: 16-byte vectors per row
    long long rowbytes;
    // workspace: [0, off_seq) holds the general path's tickets (zeroed by that
    // path at the start of every call); the rest is written by a call before the
    // same call reads it
    size_t off_c32a, off_c32b, off_seq, off_gath, off_part, off_rsum, total;
};

__host__ inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool force_generic()
{
    static const bool v = [] {
        const char* e = getenv("SPEC_VERIFY_FORCE_GENERIC");
        return e && e[0] == '1';
    }();
    return v;
}

bool make_plan(int B, int gamma, int V, sv_dtype dt, Plan* p)
{
    if (B < 1 || gamma < 1 || gamma > SV_MAX_GAMMA || V < 1 || V > SV_MAX_V) return false;
    if (dt != SV_DTYPE_F32 && dt != SV_DTYPE_BF16) return false;
    p->B = B;
    p->gamma = gamma;
    p->V = V;
    p->R = 2 * gamma + 1;
    p->esz = dt == SV_DTYPE_BF16 ? 2 : 4;
    p->rowbytes = (long long)V * p->esz;
    const long long rows = (long long)B * p->R;
    p->small = !force_generic() && V <= kSmallMaxV;
    p->stream = !force_generic() && (p->rowbytes % 16 == 0) && (p->rowbytes >= kStreamMinRowBytes);

    // generic split: ~32 KB per CTA, but at least ~2 CTAs per SM in total
    long long nc1 = cdiv(p->rowbytes, kPass1ChunkBytes);
    long long want = cdiv(2LL * kSmCount, rows);
    if (want > nc1) nc1 = want;
    long long cap = cdiv(V, kPass1MinChunk);
    if (nc1 > cap) nc1 = cap;
    if (nc1 < 1) nc1 = 1;
    p->C1 = (int)((cdiv(V, nc1) + 7) / 8 * 8);
    p->nc1 = (int)cdiv(V, p->C1);
    long long nc2 = cdiv(V, kPass2Chunk);
    want = cdiv(2LL * kSmCount, B);
    if (want > nc2) nc2 = want;
    cap = cdiv(V, kPass2MinChunk);
    if (nc2 > cap) nc2 = cap;
    if (nc2 < 1) nc2 = 1;
    p->C2 = (int)((cdiv(V, nc2) + 7) / 8 * 8);
    p->nc2 = (int)cdiv(V, p->C2);

    // streaming split: every warp span meets a row at most kStreamSlots times;
    // 512-byte tiles for the draw; the last kL2KeepBytes of the stream stay in L2
    p->nq = p->rowbytes / 16;
    p->nslot = kStreamSlots;
    p->NT2 = (int)cdiv(p->nq, kTileVecs);
    p->evict_rows = std::max<long long>(0, rows - kL2KeepBytes / p->rowbytes);

    // stream: one Partial per (row, span) slot; one float per tile (two per 8-byte slot)
    const long long nparts = rows * (p->stream ? (long long)p->nslot : p->nc1);
    const long long nrsum = p->stream ? cdiv((long long)B * p->NT2, 2) : (long long)B * p->nc2;
    size_t off = 0;
    p->off_c32a = off;  // general path: row-pass ticket per sequence
    off += sizeof(unsigned) * (size_t)B;
    p->off_c32b = off;  // general path: resample ticket per sequence
    off += sizeof(unsigned) * (size_t)B;
    off = align256(off);
    p->off_seq = off;
    off = align256(off + sizeof(SeqRec) * (size_t)B);
    p->off_gath = off;
    off = align256(off + (p->stream ? sizeof(float) * 2 * (size_t)gamma * B : 0));
    p->off_part = off;
    off = align256(off + sizeof(Partial) * (size_t)nparts);
    p->off_rsum = off;
    off = align256(off + sizeof(double) * (size_t)nrsum);
    p->total = p->small ? 256 : off;  // the small path keeps everything in registers
    return true;
}

int device_sm_count()
{
    static std::mutex mu;
    static int cache[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return kSmCount;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = kSmCount;
        cache[dev] = n;
    }
    return cache[dev];
}

// Resident CTAs per SM of a 256-thread kernel on the current device (cached per
// kernel and device; 0 on a CUDA error).
template <class K>
int ctas_per_sm(K kernel, int slot)
{
    static std::mutex mu;
    static int cache[32][kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[slot][dev]) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kPassThreads, 0) != cudaSuccess || n < 1) n = 0;
        cache[slot][dev] = n;
    }
    return cache[slot][dev];
}

// Clusters of cs CTAs of sv_draw that can be resident at once on the current
// device (cached per cluster size and device; 0 on a CUDA error).
template <int ESZ>
int max_clusters(int cs)
{
    static std::mutex mu;
    static int cache[kMaxCluster + 1][kMaxDevices] = {};
    int dev = 0;
    if (cs < 1 || cs > kMaxCluster || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[cs][dev]) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(cs * device_sm_count()));
        cfg.blockDim = dim3(kPassThreads);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)cs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, sv_draw<ESZ>, &cfg) != cudaSuccess || n < 1) n = -1;
        cache[cs][dev] = n;
    }
    return cache[cs][dev];
}

template <int ESZ, int G, int E>
cudaError_t launch_small_ge(const TailArgs& t, int B, cudaStream_t st)
{
    constexpr int slot = 2 + (G == 8 ? 0 : (G == 16 ? 4 : 8)) + (E == 1 ? 0 : (E == 2 ? 1 : (E == 4 ? 2 : 3)));
    const int c = ctas_per_sm(sv_small<ESZ, G, E>, slot + (ESZ == 4 ? 12 : 0));
    if (c < 1) return cudaErrorInvalidConfiguration;
    const long long seqs_per_cta = (long long)kWarps * (32 / G);
    const long long grid = std::min<long long>((long long)c * device_sm_count(), cdiv(B, seqs_per_cta));
    sv_small<ESZ, G, E><<<(unsigned)grid, kThreads, 0, st>>>(t, B);
    return cudaGetLastError();
}

template <int ESZ, int G>
cudaError_t launch_small_g(int E, const TailArgs& t, int B, cudaStream_t st)
{
    switch (E) {
    case 1: return launch_small_ge<ESZ, G, 1>(t, B, st);
    case 2: return launch_small_ge<ESZ, G, 2>(t, B, st);
    case 4: return launch_small_ge<ESZ, G, 4>(t, B, st);
    default: return launch_small_ge<ESZ, G, 8>(t, B, st);
    }
}

template <int ESZ>
cudaError_t launch_small(int G, int E, const TailArgs& t, int B, cudaStream_t st)
{
    if (G == 8) return launch_small_g<ESZ, 8>(E, t, B, st);
    if (G == 16) return launch_small_g<ESZ, 16>(E, t, B, st);
    return launch_small_g<ESZ, 32>(E, t, B, st);
}

template <int ESZ>
cudaError_t launch(const Plan& p, const void* tgt, const void* dft, const int32_t* tokens,
                   const float* temperature, const float* u_acc, const float* u_res, int32_t* out_tokens,
                   int32_t* out_n, double* out_ln, int32_t* out_st, unsigned char* ws, cudaStream_t st)
{
    TailArgs t;
    t.tgt = tgt;
    t.dft = dft;
    t.tokens = tokens;
    t.temperature = temperature;
    t.u_accept = u_acc;
    t.u_resample = u_res;
    t.out_tokens = out_tokens;
    t.out_n = out_n;
    t.out_log_norm = out_ln;
    t.out_status = out_st;
    t.ticket = reinterpret_cast<unsigned*>(ws + p.off_c32a);
    t.seq = reinterpret_cast<SeqRec*>(ws + p.off_seq);
    t.part = reinterpret_cast<const Partial*>(ws + p.off_part);
    t.gath = nullptr;
    t.gamma = p.gamma;
    t.V = p.V;
    t.R = p.R;

    if (p.small) {
        // groups of G lanes per sequence (the smallest of 8, 16, 32 with G >= gamma
        // and 8 * G >= V), E elements of a row per lane
        const int G = (p.gamma <= 8 && p.V <= 64) ? 8 : ((p.gamma <= 16 && p.V <= 128) ? 16 : 32);
        const int per = (int)cdiv(p.V, G);
        const int E = per <= 1 ? 1 : (per <= 2 ? 2 : (per <= 4 ? 4 : 8));
        return launch_small<ESZ>(G, E, t, p.B, st);
    }

    if (p.stream) {
        PassArgs g;
        g.t = t;
        g.part = reinterpret_cast<Partial*>(ws + p.off_part);
        g.gath = reinterpret_cast<float*>(ws + p.off_gath);
        g.t.gath = g.gath;
        g.t.nc = kStreamSlots;
        g.t.part = g.part;
        g.tsum = reinterpret_cast<float*>(ws + p.off_rsum);
        g.u_resample = u_res;
        g.nq = p.nq;
        g.NT2 = p.NT2;
        g.B = p.B;
        g.evict_rows = p.evict_rows;
        // sv_stream: as many CTAs as are resident at once, the row stream split into
        // one span per warp, each at least nq/31 vectors (a row meets at most
        // kStreamSlots spans)
        const int c1 = ctas_per_sm(sv_stream<ESZ>, ESZ == 2 ? 0 : 1);
        if (c1 < 1) return cudaErrorInvalidConfiguration;
        const long long sms = device_sm_count();
        const long long NQ = (long long)p.B * p.R * p.nq;
        const long long nw = sms * c1 * kWarps;
        g.S = std::max(std::max<long long>(kStreamSpanMin, cdiv(p.nq, kStreamSlots - 1)), cdiv(NQ, nw));
        const long long grid1 = std::min<long long>(sms * c1, cdiv(cdiv(NQ, g.S), kWarps));
        sv_stream<ESZ><<<(unsigned)grid1, kPassThreads, 0, st>>>(g);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;

        // sv_draw: clusters of cs CTAs, one sequence at a time each; the largest
        // cs (<= kMaxCluster) for which one wave of resident clusters covers the
        // batch, else 1
        int cs = 1, nclusters = 0;
        for (int c = kMaxCluster; c >= 1; c >>= 1) {
            const int n = max_clusters<ESZ>(c);
            if (n < 1) continue;
            if (c == 1 || (long long)n >= p.B) {
                cs = c;
                nclusters = n;
                break;
            }
        }
        if (nclusters < 1) return cudaErrorInvalidConfiguration;
        const long long grid2 = (long long)cs * std::min<long long>(nclusters, p.B);
        // a programmatic dependent launch: sv_draw's CTAs start as sv_stream's
        // leave, and wait on the device for sv_stream's completion
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid2);
        cfg.blockDim = dim3(kPassThreads);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)cs;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        return cudaLaunchKernelEx(&cfg, sv_draw<ESZ>, g);
    }

    // general path: zero the tickets, then the two kernels
    {
        const long long n16 = (long long)(p.off_seq / 16);
        const int gr = (int)std::min<long long>(cdiv(n16, 256), device_sm_count());
        sv_reset<<<gr, 256, 0, st>>>(reinterpret_cast<uint4*>(ws), n16);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    GenericArgs g;
    g.t = t;
    g.t.nc = p.nc1;
    g.part = reinterpret_cast<Partial*>(ws + p.off_part);
    g.nc1 = p.nc1;
    g.C1 = p.C1;
    g.u_resample = u_res;
    g.ticket2 = reinterpret_cast<unsigned*>(ws + p.off_c32b);
    g.rsum = reinterpret_cast<double*>(ws + p.off_rsum);
    g.nc2 = p.nc2;
    g.C2 = p.C2;
    const long long g1 = (long long)p.B * p.R * p.nc1;
    const long long g2 = (long long)p.B * p.nc2;
    if (g1 > 0x7fffffffLL || g2 > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    sv_rowpass<ESZ><<<(unsigned)g1, kThreads, 0, st>>>(g);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    sv_resample<ESZ><<<(unsigned)g2, kThreads, 0, st>>>(g);
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

extern "C" int spec_verify_kernels_per_call(int B, int gamma, int V, sv_dtype dt)
{
    Plan p;
    if (!make_plan(B, gamma, V, dt, &p)) return 0;
    // sv_small; sv_stream + sv_draw; or sv_reset + sv_rowpass + sv_resample
    return p.small ? 1 : (p.stream ? 2 : 3);
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
// names a stand-in, not device memory); its device address is looked up below.
//
// The address belongs to one CUDA context.  It is cached per context, keyed by
// the context's unique ID (cuCtxGetId: never reused within a process), so a
// context created later -- after cudaDeviceReset, or a caller's own context made
// current -- gets a fresh lookup instead of a stale address.  The two driver
// calls are reached through cudaGetDriverEntryPointByVersion, so the library
// does not link against the driver library.

static __device__ __align__(256) unsigned char sv_noalloc_scratch[SV_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kNoallocCache = 16;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct NoallocEntry {
    unsigned long long ctx_id;
    void* ptr;
};

std::mutex g_noalloc_mu;
NoallocEntry g_noalloc_cache[kNoallocCache] = {};
int g_noalloc_next = 0;

// Unique ID of the context current on this thread, or 0 if there is none or the
// driver calls are unavailable.
unsigned long long current_context_id()
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of sv_noalloc_scratch in the current context (the first use in a
// context does the lookup, which also makes the runtime bind a context if none is
// current).  Returns nullptr on a CUDA error.
void* noalloc_scratch_address()
{
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    unsigned long long id = current_context_id();
    if (id)
        for (const NoallocEntry& e : g_noalloc_cache)
            if (e.ctx_id == id) return e.ptr;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, sv_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    if (!id) id = current_context_id();  // the lookup may have bound the primary context
    if (id) {                            // without an ID, look it up again on every call
        g_noalloc_cache[g_noalloc_next] = NoallocEntry{id, p};
        g_noalloc_next = (g_noalloc_next + 1) % kNoallocCache;
    }
    return p;
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
    // a call reads nothing it has not written first (the general kernels' tickets
    // are zeroed by its first launch), as for any workspace
    const cudaError_t e =
        dt == SV_DTYPE_BF16
            ? launch<2>(p, target_logits, draft_logits, draft_tokens, temperature, u_accept, u_resample, out_tokens,
                        out_n_accepted, out_log_norm, out_row_status, ws, st)
            : launch<4>(p, target_logits, draft_logits, draft_tokens, temperature, u_accept, u_resample, out_tokens,
                        out_n_accepted, out_log_norm, out_row_status, ws, st);
    return e == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}

// ----------------------------------------------------------------------------- speculation cache

extern "C" sv_status spec_verify_fanout(double alpha, int gamma, int budget, int32_t* fanout)
{
    if (!fanout || gamma < 1 || gamma > SV_MAX_GAMMA || budget < 0 || !(alpha >= 0.0 && alpha <= 1.0))
        return SV_ERR_INVALID_ARG;
    // share of outcome n: alpha^n (1 - alpha), n < gamma; alpha^gamma for n = gamma
    double share[SV_MAX_GAMMA + 1];
    double an = 1.0;
    int given = 0;
    for (int n = 0; n <= gamma; ++n) {
        share[n] = (double)budget * (n < gamma ? an * (1.0 - alpha) : an);
        an *= alpha;
        fanout[n] = (int32_t)share[n];  // share >= 0: the cast rounds down
        given += fanout[n];
    }
    // the slots left over go one each to the largest remainders (smaller n first)
    while (given < budget) {
        int pick = 0;
        double most = -1.0;
        for (int n = 0; n <= gamma; ++n)
            if (share[n] - (double)fanout[n] > most) {
                most = share[n] - (double)fanout[n];
                pick = n;
            }
        ++fanout[pick];
        share[pick] -= 1.0;
        ++given;
    }
    return SV_OK;
}

namespace {

bool fill_topf_args(const int32_t* fanout, int B, int gamma, int V, sv::TopfArgs* g)
{
    if (!fanout || B < 1 || gamma < 1 || gamma > SV_MAX_GAMMA || V < 1 || V > SV_MAX_V) return false;
    g->B = B;
    g->gamma = gamma;
    g->V = V;
    g->off[0] = 0;
    g->n_nz = 0;
    for (int n = 0; n <= gamma; ++n) {
        if (fanout[n] < 0 || fanout[n] > SV_MAX_TOPF) return false;
        g->F[n] = fanout[n];
        g->off[n + 1] = g->off[n] + fanout[n];
        if (fanout[n] > 0) g->nz[g->n_nz++] = n;
    }
    g->Ftot = g->off[gamma + 1];
    return true;
}

}  // namespace

extern "C" sv_status spec_verify_topf(const void* target_logits, const void* draft_logits, sv_dtype dt,
                                      const float* temperature, const double* log_norm, const int32_t* row_status,
                                      const int32_t* fanout, int B, int gamma, int V, int32_t* out_tokens,
                                      float* out_prob, struct CUstream_st* stream)
{
    if (dt != SV_DTYPE_F32 && dt != SV_DTYPE_BF16) return SV_ERR_UNSUPPORTED_DTYPE;
    sv::TopfArgs g;
    if (!fill_topf_args(fanout, B, gamma, V, &g)) return SV_ERR_INVALID_ARG;
    if (!target_logits || !draft_logits || !temperature || !log_norm || !row_status ||
        (g.Ftot > 0 && (!out_tokens || !out_prob)))
        return SV_ERR_INVALID_ARG;
    if (!aligned(target_logits, 16) || !aligned(draft_logits, 16) || !aligned(temperature, 4) ||
        !aligned(log_norm, 8) || !aligned(row_status, 4) || !aligned(out_tokens, 4) || !aligned(out_prob, 4))
        return SV_ERR_MISALIGNED;
    if (g.n_nz == 0) return SV_OK;
    g.tgt = target_logits;
    g.dft = draft_logits;
    g.temperature = temperature;
    g.log_norm = log_norm;
    g.row_status = row_status;
    g.out_tokens = out_tokens;
    g.out_prob = out_prob;
    const unsigned grid = (unsigned)((long long)B * g.n_nz);
    cudaStream_t st = (cudaStream_t)stream;
    if (dt == SV_DTYPE_BF16) sv::sv_topf<2><<<grid, sv::kTopfThreads, 0, st>>>(g);
    else sv::sv_topf<4><<<grid, sv::kTopfThreads, 0, st>>>(g);
    return cudaGetLastError() == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}

extern "C" sv_status spec_verify_cache_lookup(const int32_t* out_tokens, const int32_t* out_n_accepted,
                                              const int32_t* cache_tokens, const int32_t* fanout, int B,
                                              int gamma, int32_t* out_slot, struct CUstream_st* stream)
{
    sv::TopfArgs g;
    if (!fill_topf_args(fanout, B, gamma, 1, &g)) return SV_ERR_INVALID_ARG;
    if (!out_tokens || !out_n_accepted || !out_slot || (g.Ftot > 0 && !cache_tokens)) return SV_ERR_INVALID_ARG;
    if (!aligned(out_tokens, 4) || !aligned(out_n_accepted, 4) || !aligned(cache_tokens, 4) || !aligned(out_slot, 4))
        return SV_ERR_MISALIGNED;
    const unsigned grid = (unsigned)cdiv(B, 256);
    sv::sv_cache_lookup<<<grid, 256, 0, (cudaStream_t)stream>>>(out_tokens, out_n_accepted, cache_tokens, g,
                                                                  out_slot);
    return cudaGetLastError() == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}

static_assert(sv::kBanditMaxArms == SV_MAX_ARMS, "arm limit");

extern "C" size_t spec_verify_bandit_state_size(int K)
{
    return (K < 1 || K > SV_MAX_ARMS) ? 0 : sizeof(double) * (size_t)(2 + 2 * K);
}

extern "C" sv_status spec_verify_bandit_init(double* state, int K, struct CUstream_st* stream)
{
    if (!state || K < 1 || K > SV_MAX_ARMS) return SV_ERR_INVALID_ARG;
    if (!aligned(state, 8)) return SV_ERR_MISALIGNED;
    sv::sv_bandit_init<<<1, 64, 0, (cudaStream_t)stream>>>(state, K);
    return cudaGetLastError() == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}

extern "C" sv_status spec_verify_bandit_step(const int32_t* n_accepted, int B, int gamma, int policy,
                                             const float* u1, const float* u2, double* state, int K,
                                             int32_t* out_arm, struct CUstream_st* stream)
{
    if (B < 0 || gamma < 1 || K < 1 || K > SV_MAX_ARMS || !state || (B > 0 && !n_accepted) ||
        (policy != SV_BANDIT_UCB1 && policy != SV_BANDIT_THOMPSON && policy != SV_BANDIT_THOMPSON_BETA) ||
        (policy != SV_BANDIT_UCB1 && (!u1 || !u2)))
        return SV_ERR_INVALID_ARG;
    if (!aligned(n_accepted, 4) || !aligned(u1, 4) || !aligned(u2, 4) || !aligned(state, 8) || !aligned(out_arm, 4))
        return SV_ERR_MISALIGNED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(sv::kBanditStepThreads);
    cfg.stream = (cudaStream_t)stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e =
        cudaLaunchKernelEx(&cfg, sv::sv_bandit_step, n_accepted, B, gamma, policy, u1, u2, state, K, out_arm);
    return e == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}

extern "C" sv_status spec_verify_bandit_simulate(const double* mu, int K, int T, int policy, int runs,
                                                 const float* uniforms, double* out_regret, double* out_state,
                                                 struct CUstream_st* stream)
{
    if (!mu || K < 1 || K > SV_MAX_ARMS || T < 0 || runs < 0 ||
        (policy != SV_BANDIT_UCB1 && policy != SV_BANDIT_THOMPSON && policy != SV_BANDIT_THOMPSON_BETA) ||
        (runs > 0 && (!uniforms || !out_regret)))
        return SV_ERR_INVALID_ARG;
    if (!aligned(mu, 8) || !aligned(uniforms, 4) || !aligned(out_regret, 8) || !aligned(out_state, 8))
        return SV_ERR_MISALIGNED;
    if (runs == 0) return SV_OK;
    constexpr int kRunsPerCta = sv::kBanditSimThreads / 32;
    const unsigned grid = (unsigned)cdiv(runs, kRunsPerCta);
    sv::sv_bandit_simulate<<<grid, sv::kBanditSimThreads, 0, (cudaStream_t)stream>>>(mu, K, T, policy, runs, uniforms,
                                                                                       out_regret, out_state);
    return cudaGetLastError() == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}

// ---------------------------------------------------------------------------- token trees

static_assert(sv::kTreeMaxNodes == SV_MAX_TREE_NODES, "tree node limit");

namespace {

// Groups of 16 bytes per row, and the cluster split: enough CTAs per tree to
// spread a row over several SMs, as long as the whole batch stays resident (two
// 512-thread CTAs per SM), and at least 512 groups (one per thread) per CTA.
void tree_plan(int B, int V, int esz, int* CL, long long* G, long long* GPC, long long* GPW)
{
    const int vec = 16 / esz;
    *G = cdiv(V, vec);
    int cl = 1;
    while (cl < sv::kTreeMaxCluster && (long long)B * cl * 2 <= 2LL * kSmCount &&
           *G / (cl * 2) >= sv::kTreeThreads)
        cl *= 2;
    *CL = cl;
    *GPC = cdiv(*G, cl);
    *GPW = cdiv(cdiv(*GPC, sv::kTreeWarps), 32) * 32;
}

}  // namespace

extern "C" sv_status spec_verify_tree(const void* target_logits, const void* draft_logits, sv_dtype dt,
                                      const int32_t* parent, const int32_t* tokens, const int32_t* keep,
                                      const float* temperature, const float* u_accept, const float* u_resample,
                                      int B, int N, int V, int32_t* out_nodes, int32_t* out_tokens,
                                      int32_t* out_n_accepted, double* out_log_norm, int32_t* out_row_status,
                                      struct CUstream_st* stream)
{
    if (dt != SV_DTYPE_F32 && dt != SV_DTYPE_BF16) return SV_ERR_UNSUPPORTED_DTYPE;
    if (B < 1 || N < 1 || N > SV_MAX_TREE_NODES || V < 1 || V > SV_MAX_V) return SV_ERR_INVALID_ARG;
    if (!target_logits || !draft_logits || !parent || !tokens || !temperature || !u_accept || !u_resample ||
        !out_nodes || !out_tokens || !out_n_accepted)
        return SV_ERR_INVALID_ARG;
    if (!aligned(target_logits, 16) || !aligned(draft_logits, 16) || !aligned(parent, 4) || !aligned(tokens, 4) ||
        !aligned(keep, 4) || !aligned(temperature, 4) || !aligned(u_accept, 4) || !aligned(u_resample, 4) ||
        !aligned(out_nodes, 4) || !aligned(out_tokens, 4) || !aligned(out_n_accepted, 4) ||
        !aligned(out_log_norm, 8) || !aligned(out_row_status, 4))
        return SV_ERR_MISALIGNED;
    const int esz = dt == SV_DTYPE_BF16 ? 2 : 4;
    sv::TreeArgs g;
    g.tgt = target_logits; g.dft = draft_logits; g.parent = parent; g.tokens = tokens; g.keep = keep;
    g.temperature = temperature; g.u_accept = u_accept; g.u_resample = u_resample;
    g.out_nodes = out_nodes; g.out_tokens = out_tokens; g.out_n = out_n_accepted;
    g.out_log_norm = out_log_norm; g.out_status = out_row_status;
    g.N = N; g.V = V;
    int CL;
    tree_plan(B, V, esz, &CL, &g.G, &g.GPC, &g.GPW);
    const bool vec16 = ((long long)V * esz) % 16 == 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((long long)B * CL));
    cfg.blockDim = dim3(sv::kTreeThreads);
    cfg.stream = (cudaStream_t)stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (dt == SV_DTYPE_BF16)
        e = vec16 ? cudaLaunchKernelEx(&cfg, sv::sv_tree<2, true>, g) : cudaLaunchKernelEx(&cfg, sv::sv_tree<2, false>, g);
    else
        e = vec16 ? cudaLaunchKernelEx(&cfg, sv::sv_tree<4, true>, g) : cudaLaunchKernelEx(&cfg, sv::sv_tree<4, false>, g);
    return e == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}

extern "C" sv_status spec_verify_tree_prune(const void* draft_logits, sv_dtype dt, const int32_t* parent,
                                            const int32_t* tokens, const float* temperature, double threshold,
                                            int B, int N, int V, int32_t* out_keep, double* out_cum,
                                            struct CUstream_st* stream)
{
    if (dt != SV_DTYPE_F32 && dt != SV_DTYPE_BF16) return SV_ERR_UNSUPPORTED_DTYPE;
    if (B < 1 || N < 1 || N > SV_MAX_TREE_NODES || V < 1 || V > SV_MAX_V || threshold != threshold)
        return SV_ERR_INVALID_ARG;
    if (!draft_logits || !parent || !tokens || !temperature || !out_keep || !out_cum) return SV_ERR_INVALID_ARG;
    if (!aligned(draft_logits, 16) || !aligned(parent, 4) || !aligned(tokens, 4) || !aligned(temperature, 4) ||
        !aligned(out_keep, 4) || !aligned(out_cum, 8))
        return SV_ERR_MISALIGNED;
    const int esz = dt == SV_DTYPE_BF16 ? 2 : 4;
    sv::PruneArgs g;
    g.dft = draft_logits; g.parent = parent; g.tokens = tokens; g.temperature = temperature;
    g.threshold = threshold; g.out_keep = out_keep; g.out_cum = out_cum;
    g.B = B; g.N = N; g.V = V;
    g.G = cdiv(V, 16 / esz);
    const bool vec16 = ((long long)V * esz) % 16 == 0;
    cudaStream_t st = (cudaStream_t)stream;
    const unsigned grid = (unsigned)((long long)B * N);
    if (dt == SV_DTYPE_BF16) {
        if (vec16) sv::sv_tree_prune_rows<2, true><<<grid, sv::kPruneThreads, 0, st>>>(g);
        else sv::sv_tree_prune_rows<2, false><<<grid, sv::kPruneThreads, 0, st>>>(g);
    } else {
        if (vec16) sv::sv_tree_prune_rows<4, true><<<grid, sv::kPruneThreads, 0, st>>>(g);
        else sv::sv_tree_prune_rows<4, false><<<grid, sv::kPruneThreads, 0, st>>>(g);
    }
    if (cudaGetLastError() != cudaSuccess) return SV_ERR_CUDA;
    sv::sv_tree_prune_walk<<<(unsigned)cdiv(B, sv::kWalkWarps), sv::kWalkWarps * 32, 0, st>>>(g);
    return cudaGetLastError() == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}

// ---------------------------------------------------------------------------- low-rank draft head

namespace {

typedef CUresult (*TensorMapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                      const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

TensorMapEncodeFn tensor_map_encoder()
{
    static TensorMapEncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<TensorMapEncodeFn>(f);
    });
    return fn;
}

// Tensor map of a row-major [rows][K] bf16 matrix, in boxes of box_k (K) x
// box_rows; out-of-range elements read as zero and are not written.
bool lr_map(CUtensorMap* m, const void* base, long long rows, long long K, int box_rows, int box_k = sv::kLrBK,
            CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B)
{
    TensorMapEncodeFn enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)box_k, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// splits > 1 (no normaliser) needs split_ws: splits * M * N floats.
template <int BN>
cudaError_t lr_launch(const void* A, const void* B, int M, int N, int K, void* out, float4* part,
                      const float* temperature, int* err, cudaStream_t st, int splits = 1, float* split_ws = nullptr)
{
    CUtensorMap ta, tb, tc;
    if (!lr_map(&ta, A, M, K, sv::kLrBM) || !lr_map(&tb, B, N, K, BN)) return cudaErrorInvalidValue;
    // the output goes out through TMA stores when its rows are 16-byte multiples
    const bool tma_store = (N % 8) == 0 && lr_map(&tc, out, M, N, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!tma_store) memset(&tc, 0, sizeof tc);
    static std::once_flag once[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    cudaError_t attr_err = cudaSuccess;
    if (dev >= 0 && dev < kMaxDevices)
        std::call_once(once[dev], [&] {
            attr_err = cudaFuncSetAttribute(sv::sv_lr_gemm<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            sv::kLrSmemMax);
        });
    if (attr_err != cudaSuccess) return attr_err;
    sv::LrArgs g;
    g.out = static_cast<__nv_bfloat16*>(out);
    g.part = part;
    g.temperature = temperature;
    g.err = err;
    g.M = M; g.N = N; g.K = K;
    g.m_tiles = (int)cdiv(M, sv::kLrBM);
    g.n_tiles = (int)cdiv(N, BN);
    const long long tiles = (long long)g.m_tiles * g.n_tiles;
    if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    const int sms = device_sm_count();
    const long long kbs = cdiv(K, sv::kLrBK);
    const long long a_bytes = (long long)sv::kLrBM * sv::kLrBK * 2, b_bytes = (long long)BN * sv::kLrBK * 2;
    const long long budget = sv::kLrSmemMax - 1024 - (tma_store ? sv::kLrStagingBytes : 0);
    // A resident: its K blocks plus at least 3 stages of B fit, and every row tile
    // gets at least one CTA
    g.tma_store = tma_store ? 1 : 0;
    g.splits = splits;
    g.part_out = split_ws;
    g.a_resident = (splits == 1 && kbs <= sv::kLrMaxResidentKb && kbs * a_bytes + 3 * b_bytes <= budget && g.m_tiles <= sms) ? 1 : 0;
    const long long stage = g.a_resident ? b_bytes : a_bytes + b_bytes;
    const long long room = budget - (g.a_resident ? kbs * a_bytes : 0);
    g.stages = (int)std::min<long long>(sv::kLrMaxStages, room / stage);
    long long grid;
    if (g.a_resident) {
        const long long slots = std::min<long long>(sms / g.m_tiles, g.n_tiles);
        grid = slots * g.m_tiles;
    } else {
        grid = std::min<long long>(tiles * splits, sms);  // one CTA per SM (shared memory)
    }
    const long long smem =
        1024 + (g.a_resident ? kbs * a_bytes : 0) + g.stages * stage + (tma_store ? sv::kLrStagingBytes : 0);
    sv::sv_lr_gemm<BN><<<(unsigned)grid, sv::kLrThreads, (size_t)smem, st>>>(ta, tb, tc, g);
    if (splits > 1) {
        if (cudaGetLastError() != cudaSuccess) return cudaErrorLaunchFailure;
        const long long total = (long long)M * N;
        const unsigned blocks = (unsigned)std::min<long long>(cdiv(total, 256), 4LL * sms);
        sv::sv_lr_splitk_sum<<<blocks, 256, 0, st>>>(split_ws, splits, M, N, static_cast<__nv_bfloat16*>(out));
    }
    return cudaGetLastError();
}

bool lr_shape_ok(int M, int d, int r, int V)
{
    // K a multiple of 8: the tensor maps' row pitch must be a multiple of 16 bytes
    return M >= 1 && d >= 8 && r >= 8 && V >= 1 && (d % 8) == 0 && (r % 8) == 0 && V <= SV_MAX_V &&
           (long long)M * r < (1LL << 40);
}

constexpr int kLrUpBN = 256;
constexpr int kLrDownBN = 64;
constexpr int kLrMaxSplits = 8;

// K slices for the down contraction inside the head: enough CTAs to fill the SMs
// when its tiles alone are few, each slice at least 4 K blocks.
int lr_down_splits(int M, int d, int r)
{
    const long long tiles = cdiv(M, sv::kLrBM) * cdiv(r, kLrDownBN);
    const long long kbs = cdiv(d, sv::kLrBK);
    long long s = std::max<long long>(1, device_sm_count() / std::max<long long>(tiles, 1));
    s = std::min<long long>(s, std::min<long long>(kLrMaxSplits, kbs / 4));
    return (int)std::max<long long>(s, 1);
}

size_t lr_u_bytes(int M, int r) { return ((size_t)M * r * 2 + 1023) / 1024 * 1024; }
size_t lr_split_bytes(int M, int r) { return ((size_t)kLrMaxSplits * M * r * 4 + 1023) / 1024 * 1024; }
size_t lr_part_bytes(int M, int V) { return (size_t)M * (size_t)cdiv(V, kLrUpBN) * sv::kLrGroups * sizeof(float4); }

}  // namespace

extern "C" size_t spec_verify_lowrank_workspace_size(int M, int r, int V)
{
    if (M < 1 || r < 8 || (r % 8) != 0 || V < 1 || V > SV_MAX_V) return 0;
    return lr_u_bytes(M, r) + lr_split_bytes(M, r) + lr_part_bytes(M, V);
}

extern "C" sv_status spec_verify_lowrank_down(const void* h, const void* w_down, int M, int d, int r, void* out_u,
                                              int32_t* out_error, struct CUstream_st* stream)
{
    if (!h || !w_down || !out_u || !lr_shape_ok(M, d, r, 1)) return SV_ERR_INVALID_ARG;
    if (!aligned(h, 16) || !aligned(w_down, 16) || !aligned(out_u, 16) || !aligned(out_error, 4))
        return SV_ERR_MISALIGNED;
    const cudaError_t e = lr_launch<kLrDownBN>(h, w_down, M, r, d, out_u, nullptr, nullptr, out_error,
                                               (cudaStream_t)stream);
    return e == cudaSuccess ? SV_OK : (e == cudaErrorInvalidValue ? SV_ERR_INVALID_ARG : SV_ERR_CUDA);
}

extern "C" sv_status spec_verify_lowrank_up(const void* u, const void* w_up, int M, int r, int V,
                                            const float* temperature, void* out_logits, double* out_lse,
                                            void* workspace, size_t workspace_bytes, int32_t* out_error,
                                            struct CUstream_st* stream)
{
    if (!u || !w_up || !out_logits || !lr_shape_ok(M, 8, r, V)) return SV_ERR_INVALID_ARG;
    if (!aligned(u, 16) || !aligned(w_up, 16) || !aligned(out_logits, 16) || !aligned(temperature, 4) ||
        !aligned(out_lse, 8) || !aligned(out_error, 4) || !aligned(workspace, 256))
        return SV_ERR_MISALIGNED;
    float4* part = nullptr;
    if (out_lse) {
        if (!workspace || workspace_bytes < lr_part_bytes(M, V)) return SV_ERR_WORKSPACE_TOO_SMALL;
        part = static_cast<float4*>(workspace);
    }
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = lr_launch<kLrUpBN>(u, w_up, M, V, r, out_logits, part, temperature, out_error, st);
    if (e != cudaSuccess) return e == cudaErrorInvalidValue ? SV_ERR_INVALID_ARG : SV_ERR_CUDA;
    if (out_lse) {
        sv::sv_lr_lse<<<(unsigned)cdiv((long long)M * 32, 256), 256, 0, st>>>(part, temperature, M,
                                                                            sv::kLrGroups * (int)cdiv(V, kLrUpBN), out_lse);
        if (cudaGetLastError() != cudaSuccess) return SV_ERR_CUDA;
    }
    return SV_OK;
}

extern "C" sv_status spec_verify_lowrank_head(const void* h, const void* w_down, const void* w_up, int M, int d,
                                              int r, int V, const float* temperature, void* out_logits,
                                              double* out_lse, void* workspace, size_t workspace_bytes,
                                              int32_t* out_error, struct CUstream_st* stream)
{
    if (!h || !w_down || !w_up || !out_logits || !lr_shape_ok(M, d, r, V)) return SV_ERR_INVALID_ARG;
    if (!workspace) return SV_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return SV_ERR_MISALIGNED;
    if (workspace_bytes < spec_verify_lowrank_workspace_size(M, r, V)) return SV_ERR_WORKSPACE_TOO_SMALL;
    void* u = workspace;
    float* split_ws = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + lr_u_bytes(M, r));
    const size_t head = lr_u_bytes(M, r) + lr_split_bytes(M, r);
    void* rest = static_cast<unsigned char*>(workspace) + head;
    if (!aligned(h, 16) || !aligned(w_down, 16)) return SV_ERR_MISALIGNED;
    // the down contraction, its K split across the SMs (its tiles alone are few)
    const cudaError_t e = lr_launch<kLrDownBN>(h, w_down, M, r, d, u, nullptr, nullptr, out_error,
                                               (cudaStream_t)stream, lr_down_splits(M, d, r), split_ws);
    if (e != cudaSuccess) return e == cudaErrorInvalidValue ? SV_ERR_INVALID_ARG : SV_ERR_CUDA;
    return spec_verify_lowrank_up(u, w_up, M, r, V, temperature, out_logits, out_lse, rest, workspace_bytes - head,
                                  out_error, stream);
}
