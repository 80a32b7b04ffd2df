// sv_bandit.cuh -- draft selection as a K-armed bandit on the device [FlashSpec,
// Metodologia 2, "Selecao de Rascunho via Bandit Online": each decoding step
// picks one draft model (an arm) from past acceptances only, the reward being
// the fraction of draft tokens accepted; UCB1 and Thompson sampling; Resultados
// Principais, "Desempenho do Bandit": the regret over T rounds].
//
// State of one bandit, caller-owned device doubles [2 + 2K]: t (rewards seen),
// the arm chosen last (-1: none yet), N_k (rewards seen for arm k), R_k (their
// sum).  A step (1) rewards the arm chosen last with the batch's accepted
// fraction sum_b n_b / (B * gamma), read straight from spec_verify's
// n_accepted, so no count crosses to the host; (2) chooses the next arm: an arm
// never rewarded (the smallest) if any, else the largest of
//   UCB1 (Auer, Cesa-Bianchi and Fischer, 2002):  R_k/N_k + sqrt(2 ln t / N_k)
//   Gaussian Thompson sampling (Agrawal and Goyal, 2013):
//       R_k/N_k + z_k / sqrt(N_k + 1),  z_k = sqrt(-2 ln(1 - u1_k)) cos(2 pi u2_k)
//       (Box-Muller on the caller's uniforms),
//   Thompson sampling with the Beta posterior's moments (uniform prior, rewards
//       in [0, 1]: Beta(R_k + 1, N_k - R_k + 1)):
//       m_k + z_k sqrt(m_k (1 - m_k) / (N_k + 3)),  m_k = (R_k + 1) / (N_k + 2),
// the smaller k on ties; a score that is NaN or -inf never wins (arm -1 when no
// score does, and the next step then rewards nothing).
//
//   sv_bandit_step      one CTA: the block sums n_accepted (int64), then lane k
//                       of warp 0 updates and scores arm k, and a shuffle
//                       reduction picks the arm.
//   sv_bandit_simulate  one warp per independent run of the regret simulation
//                       against Bernoulli arms: the same update and choice, T
//                       times, each step's uniforms loaded one step ahead.
#pragma once

#include "sv_common.cuh"

namespace sv {

constexpr int kBanditMaxArms = 16;
constexpr int kBanditStepThreads = 1024;
constexpr int kBanditSimThreads = 128;  // 4 runs per CTA
constexpr double kBanditPi = 3.141592653589793;

// Lane k < K holds arm k's N_k, R_k and uniforms; every lane of the warp returns
// the chosen arm.
__device__ __forceinline__ int bandit_choose(int K, int policy, double t, double Nk, double Rk, float u1k, float u2k)
{
    const int lane = threadIdx.x & 31;
    const bool mine = lane < K;
    const unsigned unrewarded = __ballot_sync(0xffffffffu, mine && Nk == 0.0);
    if (unrewarded) return __ffs(unrewarded) - 1;
    double score = -INFINITY;
    if (mine) {
        if (policy == 0) {
            score = Rk / Nk + sqrt(2.0 * log(t) / Nk);
        } else {
            const double z = sqrt(-2.0 * log(1.0 - (double)u1k)) * cos(2.0 * kBanditPi * (double)u2k);
            if (policy == 2) {
                const double m = (Rk + 1.0) / (Nk + 2.0);
                // multiply and add rounded apart (no fused multiply-add), as written
                score = __dadd_rn(m, __dmul_rn(z, sqrt(__dmul_rn(m, 1.0 - m) / (Nk + 3.0))));
            } else {
                score = Rk / Nk + z / sqrt(Nk + 1.0);
            }
        }
    }
    bool valid = score > -INFINITY;  // false for NaN
    int k = lane;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double os = __shfl_xor_sync(0xffffffffu, score, o);
        const int ok = __shfl_xor_sync(0xffffffffu, k, o);
        const bool ov = __shfl_xor_sync(0xffffffffu, (int)valid, o) != 0;
        if (ov && (!valid || os > score || (os == score && ok < k))) {
            score = os;
            k = ok;
            valid = true;
        }
    }
    return valid ? k : -1;
}

// Step (1) on lane k's copy of arm k: the arm chosen last earns `reward`.
__device__ __forceinline__ void bandit_reward(int arm, int K, double reward, double& t, double& Nk, double& Rk)
{
    if (arm < 0 || arm >= K) return;
    if ((int)(threadIdx.x & 31) == arm) {
        Nk += 1.0;
        Rk += reward;
    }
    t += 1.0;
}

__global__ void __launch_bounds__(kBanditStepThreads)
sv_bandit_step(const int32_t* __restrict__ n_accepted, int B, int gamma, int policy, const float* __restrict__ u1,
               const float* __restrict__ u2, double* __restrict__ state, int K, int32_t* __restrict__ out_arm)
{
    __shared__ long long s_acc[kBanditStepThreads / 32];
    // n_accepted comes from the verification launched just before on the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");
    long long acc = 0;
    for (int b = threadIdx.x; b < B; b += blockDim.x) acc += n_accepted[b];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) s_acc[warp] = acc;
    __syncthreads();
    if (warp != 0) return;
    acc = lane < (int)(blockDim.x >> 5) ? s_acc[lane] : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);

    const bool mine = lane < K;
    double t = state[0];
    const int arm = (int)state[1];
    double Nk = mine ? state[2 + lane] : 0.0;
    double Rk = mine ? state[2 + K + lane] : 0.0;
    if (B > 0) bandit_reward(arm, K, (double)acc / ((double)B * (double)gamma), t, Nk, Rk);
    const float u1k = (mine && policy != 0) ? u1[lane] : 0.0f;
    const float u2k = (mine && policy != 0) ? u2[lane] : 0.0f;
    const int pick = bandit_choose(K, policy, t, Nk, Rk, u1k, u2k);
    if (mine) {
        state[2 + lane] = Nk;
        state[2 + K + lane] = Rk;
    }
    if (lane == 0) {
        state[0] = t;
        state[1] = (double)pick;
        if (out_arm) *out_arm = pick;
    }
}

__global__ void sv_bandit_init(double* __restrict__ state, int K)
{
    const int i = threadIdx.x;
    if (i < 2 + 2 * K) state[i] = i == 1 ? -1.0 : 0.0;
}

// uniforms [runs][T + 1][2K + 1]: row s = step s's u1 (K), u2 (K), then round s's
// reward draw r.  Step 0 chooses from row 0; round s = 1..T adds the gap
// mu_max - mu[arm] of the arm in play to the regret, rewards it with
// (r_s < mu[arm]) and steps with row s.
__global__ void __launch_bounds__(kBanditSimThreads)
sv_bandit_simulate(const double* __restrict__ mu, int K, int T, int policy, int runs,
                   const float* __restrict__ uniforms, double* __restrict__ out_regret,
                   double* __restrict__ out_state)
{
    const int run = (int)((blockIdx.x * (unsigned)blockDim.x + threadIdx.x) >> 5);
    if (run >= runs) return;  // whole warps leave together: blockDim is a multiple of 32
    const int lane = threadIdx.x & 31;
    const bool mine = lane < K;
    double mu_max = mu[0];
    for (int k = 1; k < K; ++k)
        if (mu[k] > mu_max) mu_max = mu[k];
    const double muk = mine ? mu[lane] : 0.0;
    const long long row = 2 * K + 1;
    const float* u = uniforms + (long long)run * (T + 1) * row;

    double t = 0.0, Nk = 0.0, Rk = 0.0, regret = 0.0;
    int arm = bandit_choose(K, policy, t, Nk, Rk, mine ? u[lane] : 0.0f, mine ? u[K + lane] : 0.0f);
    // the next row's values, loaded one step ahead
    float n1 = 0.0f, n2 = 0.0f, nr = 0.0f;
    if (T >= 1) {
        const float* us = u + row;
        n1 = mine ? us[lane] : 0.0f;
        n2 = mine ? us[K + lane] : 0.0f;
        nr = us[2 * K];
    }
    for (int s = 1; s <= T; ++s) {
        const float c1 = n1, c2 = n2, cr = nr;
        if (s < T) {
            const float* us = u + (long long)(s + 1) * row;
            n1 = mine ? us[lane] : 0.0f;
            n2 = mine ? us[K + lane] : 0.0f;
            nr = us[2 * K];
        }
        if (arm >= 0) {
            const double mu_arm = __shfl_sync(0xffffffffu, muk, arm);
            regret += mu_max - mu_arm;
            const int reward = (double)cr < mu_arm ? 1 : 0;
            bandit_reward(arm, K, (double)reward, t, Nk, Rk);  // one sequence, gamma = 1
        }
        arm = bandit_choose(K, policy, t, Nk, Rk, c1, c2);
    }
    if (lane == 0) out_regret[run] = regret;
    if (out_state) {
        double* o = out_state + (long long)run * (2 + 2 * K);
        if (lane == 0) {
            o[0] = t;
            o[1] = (double)arm;
        }
        if (mine) {
            o[2 + lane] = Nk;
            o[2 + K + lane] = Rk;
        }
    }
}

}  // namespace sv
