/*
 * spec_verify.h -- C ABI of the B200 batched speculative-sampling verifier.
 *
 * One call verifies B independent sequences, each carrying gamma draft tokens,
 * entirely on the GPU with no host synchronisation.  The on-device accept /
 * reject decision replaces a per-step device-to-host copy whose cost grows with
 * the vocabulary size [FlashSpec (gist.science rs-10162738), "Declaracao do
 * Problema" 1 and Metodologia 1, "Kernel de Verificacao no Dispositivo"].
 *
 * For every sequence b with temperature T = temperature[b] > 0:
 *   1. Both models' logits are scaled by 1/T before the log-softmax, and every
 *      row is normalised in log space over the whole vocabulary V in one
 *      streaming pass [FlashSpec, Metodologia 1, "Estabilidade Numerica";
 *      "Significancia", engineering lessons]:
 *          lse(row) = log sum_v exp(l_v / T)
 *   2. For each draft position j the kernel reads two log-probability scalars,
 *          log p_j(x_j) = lt[b][j][x_j]/T - lse_t[j],
 *          log q_j(x_j) = ld[b][j][x_j]/T - lse_d[j]
 *      [FlashSpec, Metodologia 1, "Mecanismo"], and accepts x_j iff
 *          log u_accept[b][j] < log p_j(x_j) - log q_j(x_j).
 *      The accepted prefix ends at the first rejection n (n = gamma if none)
 *      and the rest of the draft is dropped [Speculative Speculative Decoding
 *      (gist.science 2603.03251), "O Essencial", step 3].
 *   3. The outcome is n plus one more token [Speculative Speculative Decoding,
 *      Metodologia 2, "Conceito Central" 1]: after a rejection it is drawn from
 *      the residual distribution norm(max(0, p_n - q_n)) [same page, Desafios 2,
 *      "Amostragem Saguaro"]; after gamma acceptances it is the bonus token,
 *      drawn from the target's (gamma+1)-th distribution p_gamma.  The draw is
 *      an inverse CDF with u = u_resample[b]: the smallest token k whose running
 *      weight sum C_k exceeds u * (sum of all weights).  A residual whose total
 *      mass is below 2^-18 counts as vanished (q_n equals p_n to within
 *      rounding there, and the residual is then proportional to p_n): the token
 *      is drawn from p_n and status bit SV_ROW_RESIDUAL_ZERO is set.
 * With T == 0 the step is greedy: x_j is accepted iff it is the first argmax of
 * target row j, and the extra token is the first argmax of target row n.  The
 * draft logits and the uniforms of such a sequence are not read.
 *
 * The uniforms are inputs, so a call is a deterministic function of its
 * arguments and can be reproduced bit for bit.
 *
 * Numerics: the normaliser sums are accumulated in fp32 from exact bf16/fp32
 * inputs and finished in fp64; the accept test runs in fp64.  Compared with an
 * exact evaluation, a decision can differ only when |log u - (log p - log q)|
 * or the inverse-CDF gap to u is below ~1e-6.
 */
#ifndef SPEC_VERIFY_H_
#define SPEC_VERIFY_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so C callers need no CUDA header. */
struct CUstream_st;

typedef enum {
    SV_OK = 0,
    SV_ERR_INVALID_ARG = 1,        /* bad size, null required pointer, bad enum */
    SV_ERR_UNSUPPORTED_DTYPE = 2,  /* dt is not SV_DTYPE_F32 / SV_DTYPE_BF16 */
    SV_ERR_MISALIGNED = 3,         /* logits not 16-byte aligned, or a pointer not
                                      aligned to its element / workspace to 256 bytes */
    SV_ERR_WORKSPACE_TOO_SMALL = 4,/* workspace_bytes < spec_verify_workspace_size() */
    SV_ERR_CUDA = 5                /* a CUDA launch or runtime call failed */
} sv_status;

typedef enum { SV_DTYPE_F32 = 0, SV_DTYPE_BF16 = 1 } sv_dtype;

/* Limits checked on the host before anything is launched. */
#define SV_MAX_GAMMA 32
#define SV_MAX_V (1 << 30)
/* Smallest positive temperature; 0 < T < SV_TEMPERATURE_MIN counts as invalid. */
#define SV_TEMPERATURE_MIN 1e-6f

/* Per-sequence status bits written to out_row_status (data-dependent errors
 * never trap; they are reported here).  With bit 1, 2, 4 or 16 the sequence
 * emits n_accepted = 0 and out_tokens all -1. */
#define SV_ROW_BAD_TOKEN 1        /* some draft token outside [0, V) */
#define SV_ROW_BAD_LOGITS 2       /* a row that is read holds NaN or +inf, or is all -inf */
#define SV_ROW_BAD_TEMPERATURE 4  /* T < 0, NaN, +inf, or 0 < T < SV_TEMPERATURE_MIN */
#define SV_ROW_RESIDUAL_ZERO 8    /* residual mass below 2^-18 (it counts as vanished);
                                     the token was drawn from p_n instead */
#define SV_ROW_BAD_UNIFORM 16     /* T > 0 and some u_accept[b][j] or u_resample[b]
                                     outside [0, 1) or NaN */
#define SV_ROW_BAD_TREE 32        /* spec_verify_tree: a parent index out of range */

/*
 * Bytes of device workspace spec_verify() needs for this shape (0 on a bad
 * shape).  The workspace is caller-owned device memory, 256-byte aligned.
 * Infrastructure of this library: no passage of the pages stands behind it.
 *
 * The workspace needs no initialisation and keeps nothing between calls: a call
 * reads no byte of it that the same call has not written first (the general
 * kernels' per-sequence tickets are zeroed by the call's first launch), so any
 * contents -- another shape's leftovers, garbage -- are fine.  Calls that share
 * a workspace must be ordered (same stream, or events).  No kernel of either
 * family waits on another, so there is no timeout or error word.
 */
size_t spec_verify_workspace_size(int B, int gamma, int V, sv_dtype dt);

/* Number of kernel launches one spec_verify() call of this shape enqueues: 1
 * for rows of at most 256 elements (8, 16 or 32 lanes per sequence), 2 for 16-byte-aligned
 * rows of at least 4 KB (the streaming pass, then the draw), 3 otherwise (ticket
 * reset, row pass, resample); 0 on a bad shape.  Infrastructure: no passage of
 * the pages stands behind it. */
int spec_verify_kernels_per_call(int B, int gamma, int V, sv_dtype dt);

/* cudaMemsetAsync(workspace, 0, workspace_bytes, stream).  Not required before
 * spec_verify (see spec_verify_workspace_size); kept for callers that want a
 * known state.  Infrastructure: no passage of the pages stands behind it. */
sv_status spec_verify_workspace_init(void* workspace, size_t workspace_bytes,
                                     struct CUstream_st* stream);

/*
 * Verify B sequences.  All pointers are caller-owned DEVICE memory on the
 * current device; the library allocates nothing, keeps no state between calls
 * and does not synchronise with the host.  Work is enqueued on `stream` and the
 * call returns right after the enqueue; results are visible to later work on
 * that stream.
 *
 *   target_logits   [B][gamma+1][V] of dt, contiguous, 16-byte aligned
 *   draft_logits    [B][gamma][V]   of dt, contiguous, 16-byte aligned
 *   draft_tokens    [B][gamma] int32
 *   temperature     [B] float; 0 = greedy
 *   u_accept        [B][gamma] float in [0, 1) (else status SV_ROW_BAD_UNIFORM)
 *   u_resample      [B] float in [0, 1) (else status SV_ROW_BAD_UNIFORM)
 *   out_tokens      [B][gamma+1] int32: the n accepted drafts, the extra token,
 *                   then -1
 *   out_n_accepted  [B] int32 in [0, gamma]
 *   workspace       see spec_verify_workspace_size()
 *   out_log_norm    optional [B][2*gamma+1] double: lse of the target rows, then
 *                   the draft rows; NaN for greedy or invalid sequences and bad rows
 *   out_row_status  optional [B] int32 bitmask of SV_ROW_* (0 = ok)
 *
 * Returns SV_OK after a successful enqueue.  Host-checkable errors return before
 * anything is launched and leave every output untouched.  SV_ERR_CUDA reports a
 * failed launch; outputs are then undefined.
 */
sv_status spec_verify(const void* target_logits, const void* draft_logits, sv_dtype dt,
                      const int32_t* draft_tokens, const float* temperature,
                      const float* u_accept, const float* u_resample,
                      int32_t* out_tokens, int32_t* out_n_accepted,
                      int B, int gamma, int V,
                      void* workspace, size_t workspace_bytes,
                      double* out_log_norm, int32_t* out_row_status,
                      struct CUstream_st* stream);

/* Static description of a status code; never NULL.  Infrastructure: no passage
 * of the pages stands behind it. */
const char* spec_verify_status_string(sv_status status);

/*
 * No-allocation variant.  The pages have no counterpart to this entry point;
 * it exists for callers that must not allocate device memory themselves: code
 * running inside another runtime's enqueue hook (an inference-engine plugin,
 * for example) or under a fixed memory budget owned by someone else, where a
 * cudaMalloc is forbidden or would synchronise the device in the middle of a
 * decode step.
 *
 * Same arguments and results as spec_verify(), minus the workspace: the
 * scratch lives in a fixed device array inside this library,
 * SV_NOALLOC_SCRATCH_BYTES bytes on every GPU that loads the library, held
 * until the process exits.  The caller still passes every input and output.
 *
 *  - Shapes whose workspace (spec_verify_workspace_size) exceeds
 *    SV_NOALLOC_SCRATCH_BYTES are rejected with SV_ERR_WORKSPACE_TOO_SMALL
 *    before anything is launched.
 *  - The first call in a CUDA context (a device's primary context, or a context
 *    the caller made current) looks up the array's device address in that
 *    context; make that first call before any stream capture begins.  The
 *    address is cached per context under the context's unique ID, so after
 *    cudaDeviceReset, or in another context, the next call looks it up again
 *    rather than reusing an address that no longer belongs to it.
 *  - The call allocates nothing: it launches the same kernels as spec_verify()
 *    on `stream`, the first of which zeroes the counters in the array.
 *  - Every call shares the one array and leaves its contents behind, so calls
 *    that overlap on the GPU (different streams without ordering, or several
 *    host threads) race and give wrong results.  Order them.
 */
#define SV_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)

sv_status spec_verify_noalloc(const void* target_logits, const void* draft_logits, sv_dtype dt,
                              const int32_t* draft_tokens, const float* temperature,
                              const float* u_accept, const float* u_resample,
                              int32_t* out_tokens, int32_t* out_n_accepted,
                              int B, int gamma, int V,
                              double* out_log_norm, int32_t* out_row_status,
                              struct CUstream_st* stream);

/*
 * ---------------------------------------------------------------------------
 * The speculation cache's side of an outcome [Speculative Speculative
 * Decoding, Metodologia 2, "Conceito Central": a verification outcome is the
 * number of accepted drafts plus one more token, and the cache holds
 * speculations for likely outcomes; Desafios 1: a geometric fan-out of cache
 * slots over the accepted lengths within a budget; Desafios 2: the extra token
 * after a rejection follows the residual distribution, and the cached tokens
 * are its most probable ones].
 */

/* Most cache slots one outcome can have in spec_verify_topf. */
#define SV_MAX_TOPF 32

/* Cache slots per outcome n in [0, gamma], on the host: outcome n has share
 * alpha^n (1 - alpha) (n < gamma) or alpha^gamma (n = gamma) of the budget -- the
 * law of the accepted length when each position accepts with probability alpha
 * -- rounded down, and the slots left over go one each to the largest
 * remainders (the smaller n on ties).  fanout: host int32[gamma + 1].
 * Returns SV_ERR_INVALID_ARG for alpha outside [0, 1], gamma outside
 * [1, SV_MAX_GAMMA], a negative budget or a null pointer. */
sv_status spec_verify_fanout(double alpha, int gamma, int budget, int32_t* fanout);

/*
 * For every sequence b and outcome n with fanout[n] > 0, the fanout[n] most
 * probable tokens of the distribution spec_verify draws the extra token from
 * after outcome n: norm(max(0, p_n - q_n)) for n < gamma (p_n when that residual
 * mass is below 2^-18, as spec_verify does), p_gamma for n = gamma, and for
 * T = 0 a point mass on the first argmax of target row n; in decreasing
 * probability, equal probabilities smaller token first, with the probabilities.
 * Slots past the tokens of positive probability hold -1 and 0; sequences whose
 * row_status has SV_ROW_BAD_TEMPERATURE or SV_ROW_BAD_LOGITS hold -1 and 0
 * everywhere.  Outcome n's slots are [off_n, off_n + fanout[n]) of each row,
 * off_n = fanout[0] + ... + fanout[n-1].
 *
 *   target_logits, draft_logits, dt, temperature  as for spec_verify
 *   log_norm      [B][2*gamma+1] double and row_status [B] int32: spec_verify's
 *                 out_log_norm and out_row_status for the same inputs (p and q
 *                 are formed from these normalisers: one pass over the rows)
 *   fanout        HOST int32[gamma + 1], each in [0, SV_MAX_TOPF]
 *   out_tokens    [B][sum fanout] int32;  out_prob [B][sum fanout] float
 *
 * Device pointers are caller-owned; nothing is allocated, no workspace.
 * Host-checkable errors return before any launch.  Infrastructure around the
 * passages above; the selection rule (most probable first, smaller token on
 * ties) is this library's reading.
 */
sv_status spec_verify_topf(const void* target_logits, const void* draft_logits, sv_dtype dt,
                           const float* temperature, const double* log_norm, const int32_t* row_status,
                           const int32_t* fanout, int B, int gamma, int V, int32_t* out_tokens,
                           float* out_prob, struct CUstream_st* stream);

/*
 * Whether each sequence's outcome is in its cache: out_slot[b] = the first slot
 * s of outcome n's range (n = out_n_accepted[b]) with cache_tokens[b][s] equal to
 * the extra token out_tokens[b][n], else -1 (also when that token is -1).
 *   out_tokens [B][gamma+1], out_n_accepted [B]: spec_verify's outputs;
 *   cache_tokens [B][sum fanout] (e.g. spec_verify_topf's out_tokens);
 *   fanout HOST int32[gamma + 1]; out_slot [B] int32.  All device pointers but
 *   fanout.
 */
sv_status spec_verify_cache_lookup(const int32_t* out_tokens, const int32_t* out_n_accepted,
                                   const int32_t* cache_tokens, const int32_t* fanout, int B, int gamma,
                                   int32_t* out_slot, struct CUstream_st* stream);

/*
 * ---------------------------------------------------------------------------
 * Draft selection as a K-armed bandit, on the device [FlashSpec, Metodologia 2,
 * "Selecao de Rascunho via Bandit Online": each decoding step picks one of K
 * draft models (arms) from past acceptances only; the reward is the fraction of
 * draft tokens accepted; UCB1 and Thompson sampling.  Resultados Principais,
 * "Desempenho do Bandit": regret over T rounds].  The reward is summed from
 * spec_verify's out_n_accepted on the device, so no per-sequence count crosses
 * to the host; the chosen arm is one int32 in device memory.
 *
 * State (caller-owned device doubles, spec_verify_bandit_state_size(K) bytes):
 *   [0] t = rewards seen, [1] the arm chosen last (-1: none yet),
 *   [2, 2+K) N_k = rewards seen for arm k, [2+K, 2+2K) R_k = their sum.
 * The state is the only memory a bandit keeps; steps on one state must be
 * ordered (same stream, or events).
 */
#define SV_MAX_ARMS 16
#define SV_BANDIT_UCB1 0
#define SV_BANDIT_THOMPSON 1
#define SV_BANDIT_THOMPSON_BETA 2

/* Bytes of one bandit's state, 8 * (2 + 2K); 0 for K outside [1, SV_MAX_ARMS]. */
size_t spec_verify_bandit_state_size(int K);

/* Enqueue writing the empty state (t = 0, arm = -1, N = R = 0) to `state`
 * (device, 8-byte aligned). */
sv_status spec_verify_bandit_init(double* state, int K, struct CUstream_st* stream);

/*
 * One decoding step of the bandit:
 *  (1) if an arm in [0, K) was chosen last and B > 0, it earns the reward
 *      sum_b n_accepted[b] / (B * gamma) (the batch's accepted fraction, summed
 *      exactly in 64-bit integers, divided in fp64): N_arm += 1, R_arm += reward,
 *      t += 1;
 *  (2) the next arm: the smallest arm never rewarded (N_k = 0) if any; else the
 *      largest score, the smaller k on ties, where
 *        SV_BANDIT_UCB1 (Auer, Cesa-Bianchi and Fischer, 2002):
 *            R_k/N_k + sqrt(2 ln t / N_k)
 *        SV_BANDIT_THOMPSON, Gaussian posteriors (Agrawal and Goyal, 2013):
 *            R_k/N_k + z_k / sqrt(N_k + 1),
 *            z_k = sqrt(-2 ln(1 - u1[k])) cos(2 pi u2[k])   (Box-Muller);
 *        SV_BANDIT_THOMPSON_BETA, a normal draw with the moments of the Beta
 *            posterior Beta(R_k + 1, N_k - R_k + 1) (uniform prior):
 *            m_k + z_k sqrt(m_k (1 - m_k) / (N_k + 3)),  m_k = (R_k + 1)/(N_k + 2);
 *      a score that is NaN or -inf never wins; when none wins the arm is -1 and
 *      the next step rewards nothing.
 *  (3) state[1] and *out_arm (if not null) = that arm.
 *
 *   n_accepted  [B] int32 (spec_verify's out_n_accepted); B = 0 rewards nothing
 *   u1, u2      [K] float in [0, 1), this step's uniforms; read for the two
 *               Thompson policies only (may be null for UCB1)
 *   state       as above;  out_arm  optional [1] int32
 * All pointers are device memory.  The kernel waits (programmatic dependent
 * launch) for the work before it on the stream, so it can follow spec_verify
 * directly.  Returns SV_ERR_INVALID_ARG for K outside [1, SV_MAX_ARMS], B < 0,
 * gamma < 1, an unknown policy or a missing pointer, before any launch.
 * Scores are fp64 (log, cos, sqrt of the CUDA math library): compared with an
 * exact evaluation a choice can differ only between arms whose scores agree to
 * within a few units in the last place.  The unrewarded-first rule and the
 * Gaussian form of the Thompson posterior are this library's readings.
 */
sv_status spec_verify_bandit_step(const int32_t* n_accepted, int B, int gamma, int policy,
                                  const float* u1, const float* u2, double* state, int K,
                                  int32_t* out_arm, struct CUstream_st* stream);

/*
 * The regret simulation: `runs` independent bandits, each played for T rounds
 * against K Bernoulli arms of means mu[k], with one sequence and gamma = 1 per
 * step (a reward is 0 or 1).  uniforms [runs][T+1][2K+1] float: row s holds
 * step s's u1 (K values), u2 (K values), then round s's reward draw r_s.  Step 0
 * (nothing to reward) chooses from row 0; round s = 1..T adds the gap
 * max_k mu_k - mu[arm] of the arm in play to the run's regret, rewards that arm
 * with (r_s < mu[arm]) and steps with row s.
 *   out_regret [runs] double;  out_state optional [runs][2+2K] double: each
 *   run's final state.  mu [K] double.  All device pointers.
 */
sv_status spec_verify_bandit_simulate(const double* mu, int K, int T, int policy, int runs,
                                      const float* uniforms, double* out_regret, double* out_state,
                                      struct CUstream_st* stream);

/*
 * ---------------------------------------------------------------------------
 * Token trees [SpecLA, Metodologia 1, "Kernels de Verificacao de Topologia
 * Conscientes": drafts shaped as chains or as branching trees; Metodologia 3,
 * "Poda Guiada por Confianca": paths of low cumulative draft log-probability are
 * removed before verification; Speculative Speculative Decoding, "Significado e
 * Impacto": the method is compatible with token trees].
 *
 * Layout of sequence b with N nodes: node 0 is the root (the context verified
 * so far); node i >= 1 carries a draft token tokens[b][i] and a parent
 * parent[b][i] in [0, i) (parent[b][0] = -1), so parents come before children.
 * target_logits [B][N][V] hold the target's next-token logits at node i's
 * context (the path to i, tokens[b][i] included), draft_logits [B][N][V] the
 * draft's there (the distribution node i's children were drawn from).
 */
#define SV_MAX_TREE_NODES 64

/*
 * Verify B token trees.  The pages give no rule for several candidates; this is
 * the multi-candidate form of spec_verify's test (its output law is the
 * target's when the children of a node are independent draws from q there):
 * at node c (first the root) P is the target's p at c; the children of c that
 * take part are tested in increasing index, child i accepted iff
 *     log u_accept[b][i] < log P(x_i) - log q_c(x_i);
 * after a rejection P becomes norm(max(0, P - q_c)) (or stays P when that mass
 * is below 2^-18: status bit SV_ROW_RESIDUAL_ZERO); an accepted child becomes c;
 * when no child of c is accepted, or c has none, the extra token is drawn from P
 * by spec_verify's inverse CDF with u_resample[b].  T = 0: the first child whose
 * token is the first argmax of target row c is accepted, else that argmax is the
 * extra token.  On a chain (parent i - 1) the result is spec_verify's.
 *
 *   keep            optional [B][N] int32: node i >= 1 takes part iff keep != 0
 *                   and its parent takes part (spec_verify_tree_prune's output)
 *   u_accept        [B][N] float (entry 0 unused);  u_resample [B] float
 *   out_nodes       [B][N] int32: the accepted nodes in path order, then -1
 *   out_tokens      [B][N] int32: their tokens, the extra token, then -1
 *   out_n_accepted  [B] int32: the number of accepted nodes (path depth)
 *   out_log_norm    optional [B][2N] double: lse of target row i at [i], of draft
 *                   row i at [N + i], for the rows the walk read; NaN elsewhere
 *   out_row_status  optional [B] int32: SV_ROW_* bits.  The walk reads target row
 *                   c of every node c it visits and (T > 0) draft row c when c has
 *                   children taking part; status 2 only for a bad row among them.
 *                   Status 1 / 16 concern the nodes that take part; 32 a parent
 *                   index out of range.  With 1, 2, 4, 16 or 32 nothing is emitted.
 *
 * All pointers are caller-owned device memory (the logits 16-byte aligned);
 * nothing is allocated and no workspace is needed; one launch (a cluster of up
 * to 8 CTAs per tree).  Host-checkable errors (N outside [1,
 * SV_MAX_TREE_NODES], V outside [1, SV_MAX_V], B < 1, a null pointer, a bad
 * dtype, misalignment) return before any launch.
 */
sv_status spec_verify_tree(const void* target_logits, const void* draft_logits, sv_dtype dt,
                           const int32_t* parent, const int32_t* tokens, const int32_t* keep,
                           const float* temperature, const float* u_accept, const float* u_resample,
                           int B, int N, int V, int32_t* out_nodes, int32_t* out_tokens,
                           int32_t* out_n_accepted, double* out_log_norm, int32_t* out_row_status,
                           struct CUstream_st* stream);

/*
 * Pruning by path probability, before verification: for node i >= 1 with parent c
 *     out_cum[b][i] = out_cum[b][c] + log q_c(tokens[b][i]),  out_cum[b][0] = 0,
 * log q_c = the draft's log-softmax of row c at temperature T (T = 0: 0 at the
 * first argmax of draft row c, -inf elsewhere), and
 *     out_keep[b][i] = out_keep[b][c] and not (out_cum[b][i] < threshold).
 * Where the sum cannot be formed (a bad temperature or parent index: every node
 * of the sequence; a token outside [0, V) or a bad draft row: that node and what
 * adds to it) out_cum is NaN and the node is kept, so spec_verify_tree reports
 * the fault.  Pruning chooses the proposals: spec_verify_tree's output law is
 * the target's only for children drawn independently from q, which a
 * threshold on their own probability is not (greedy trees excepted).
 *   out_keep [B][N] int32, out_cum [B][N] double.  Two launches.
 */
sv_status spec_verify_tree_prune(const void* draft_logits, sv_dtype dt, const int32_t* parent,
                                 const int32_t* tokens, const float* temperature, double threshold, int B,
                                 int N, int V, int32_t* out_keep, double* out_cum, struct CUstream_st* stream);

/*
 * ---------------------------------------------------------------------------
 * The low-rank draft head [SlimSpec, Metodologia, "Arquitetura": the draft's LM
 * head z = W_up W_down h with W_down in R^{r x d} and W_up in R^{V x r}, r << d
 * (e.g. d/8), in place of the full-rank W_full h], producing the draft logits the
 * verifier reads, on the tensor cores (tcgen05, bf16 in, fp32 accumulation).
 *
 * All matrices are bf16, row-major, K-major as stored:
 *   h [M][d] (one row per draft position: M = B * gamma), W_down [r][d],
 *   W_up [V][r]; d and r multiples of 8; every pointer 16-byte aligned.
 *   u [M][r] = bf16(h W_down^T)   (the intermediate is rounded to bf16: the
 *                                  second contraction takes bf16 operands)
 *   z [M][V] = bf16(u W_up^T)     (the draft logits)
 *   out_lse [M] (optional): the log-normaliser of each row of z at temperature
 *   temperature[m] (null: 1), the value spec_verify's out_log_norm gives for that
 *   draft row; NaN for T = 0 or an invalid T, and for a row with NaN or +inf.
 * out_error (optional, device int32): set to 1 if a kernel gave up waiting on its
 * own pipeline (outputs are then undefined); never set on a working GPU.
 * Host-checkable errors return before any launch.
 */

/* Workspace bytes of spec_verify_lowrank_head (u and the normaliser partials);
 * spec_verify_lowrank_up needs lowrank_workspace_size minus the u part, only when
 * out_lse is requested.  0 on a bad shape. */
size_t spec_verify_lowrank_workspace_size(int M, int r, int V);

/* u = bf16(h W_down^T): [M][r]. */
sv_status spec_verify_lowrank_down(const void* h, const void* w_down, int M, int d, int r, void* out_u,
                                   int32_t* out_error, struct CUstream_st* stream);

/* z = bf16(u W_up^T): [M][V], and (if out_lse) each row's log-normaliser; the
 * workspace (256-byte aligned) holds the normaliser partials:
 * spec_verify_lowrank_workspace_size(M, r, V) minus the u part. */
sv_status spec_verify_lowrank_up(const void* u, const void* w_up, int M, int r, int V, const float* temperature,
                                 void* out_logits, double* out_lse, void* workspace, size_t workspace_bytes,
                                 int32_t* out_error, struct CUstream_st* stream);

/* Both contractions: the head from h to the draft logits (and normalisers).  The
 * down contraction's K is split across the SMs when its tiles alone are few (its
 * fp32 slices, kept in the workspace, are added in slice order and rounded to
 * bf16 once). */
sv_status spec_verify_lowrank_head(const void* h, const void* w_down, const void* w_up, int M, int d, int r,
                                   int V, const float* temperature, void* out_logits, double* out_lse,
                                   void* workspace, size_t workspace_bytes, int32_t* out_error,
                                   struct CUstream_st* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPEC_VERIFY_H_ */
