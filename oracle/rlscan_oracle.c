/*
 * rlscan oracle: plain, slow, sequential fp64 reference for the seven RL
 * credit-assignment estimators.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may call,
 * link or load this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA library.
 *
 * Source of each definition: "rl-triton" project README
 * (deploy-preview-8--rl-triton.netlify.app), section "Kernels" (one row per
 * estimator) and the with-truncations paragraph under "Performance"; the
 * arXiv abstract of "rl-triton: High-Performance Triton GPU Kernels for
 * Reinforcement Learning Credit Assignment" (arXiv:2608.17641), which states
 * that every estimator is one first-order linear recurrence and that
 * terminated and truncated episodes are treated explicitly.  The pages give
 * the eligibility-trace formula only; the others are the textbook
 * definitions named in each function's comment.
 *
 * Conventions (the readings of the pages this oracle encodes):
 *   - every array is row-major [E][T] (Retrace's per-action arrays [E][T][A]),
 *     T contiguous; inputs are float32, outputs float64;
 *   - a flag (terminated, truncated, done) is true iff it is nonzero;
 *   - terminated at t: the episode ends at t with no bootstrap and the trace
 *     is cut; truncated at t: the episode ends at t, its value is
 *     bootstrapped with bootstrap_values[t] and the trace is cut; when both
 *     are set, terminated wins;
 *   - the value after the last step of a row (t = T-1, no flag) is
 *     last_values[e], or 0 when last_values is NULL;
 *   - forward estimators reset after a done: d[t-1] != 0 starts a new
 *     episode at t.  The README's trace formula writes (1-d) without a
 *     subscript, so its other reading, d[t] != 0 marks t itself as the first
 *     step of an episode, is the `done_starts_episode` argument;
 *   - a cut trace is a branch, not a multiplication by zero, so a non-finite
 *     value never leaks across an episode boundary.
 * All arithmetic is fp64 on the fp32 inputs widened exactly.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)

static int is_set(const float *flags, int64_t i)
{
    return flags != NULL && flags[i] != 0.0f;
}

/* Episode status of step i: *cont = episode goes on after i (no flag set),
 * *trn = episode was truncated at i (and not terminated). */
static void step_status(const float *term, const float *trunc, int64_t i,
                        int *cont, int *trn)
{
    int te = is_set(term, i);
    int tr = is_set(trunc, i) && !te;
    *cont = !te && !tr;
    *trn = tr;
}

static double last_value(const float *last_values, int64_t e)
{
    return last_values != NULL ? (double)last_values[e] : 0.0;
}

/* Value that the TD error at step i bootstraps from: V(next state) when the
 * episode goes on, bootstrap_values[i] at a truncation, 0 at a termination. */
static double bootstrap(int cont, int trn, double next_value, const float *bv,
                        int64_t i)
{
    if (cont)
        return next_value;
    if (trn)
        return (double)bv[i];
    return 0.0;
}

static int check_common(const void *a, const void *b, int64_t E, int64_t T)
{
    if (E < 0 || T < 0)
        return ORACLE_EINVAL;
    if ((E > 0 && T > 0) && (a == NULL || b == NULL))
        return ORACLE_EINVAL;
    return ORACLE_OK;
}

/*
 * GAE (README "Kernels": "backward scan over delta + gamma*lambda*A";
 * Schulman et al. 2016, the GAE(gamma, lambda) sum in recursive form):
 *   delta_t = r_t + gamma * boot_t - V_t
 *   A_t     = delta_t + gamma*lambda * A_{t+1}   while the episode goes on,
 *   A_t     = delta_t                            at a terminated/truncated step,
 * with A_T = 0 and boot_t = V_{t+1} (V_T = last value), bootstrap_values[t]
 * at a truncation, 0 at a termination.
 */
int oracle_gae(const float *rewards, const float *values, const float *terminateds,
               const float *truncateds, const float *bootstrap_values,
               const float *last_values, double *advantages, int64_t E, int64_t T,
               double gamma, double lambda_)
{
    if (check_common(rewards, values, E, T) || (E > 0 && T > 0 && advantages == NULL))
        return ORACLE_EINVAL;
    if (truncateds != NULL && bootstrap_values == NULL)
        return ORACLE_EINVAL;
    for (int64_t e = 0; e < E; ++e) {
        const int64_t row = e * T;
        double a_next = 0.0;
        for (int64_t t = T - 1; t >= 0; --t) {
            const int64_t i = row + t;
            int cont, trn;
            step_status(terminateds, truncateds, i, &cont, &trn);
            double next_v = (t + 1 < T) ? (double)values[i + 1] : last_value(last_values, e);
            double delta = (double)rewards[i] + gamma * bootstrap(cont, trn, next_v, bootstrap_values, i)
                           - (double)values[i];
            double adv = cont ? delta + gamma * lambda_ * a_next : delta;
            advantages[i] = adv;
            a_next = adv;
        }
    }
    return ORACLE_OK;
}

/*
 * V-Trace (README "Kernels": "IS-weighted targets and advantages"; Espeholt
 * et al. 2018, IMPALA, section 4.1 (the v-trace target), with the
 * lambda-weighted trace c_t = lambda * min(c_bar, pi/mu) that section remarks on):
 *   rho_t = min(rho_bar, exp(log_rho_t)),  c_t = lambda * min(c_bar, exp(log_rho_t))
 *   D_t   = rho_t (r_t + gamma*boot_t - V_t) + gamma c_t D_{t+1}  (trace cut at flags)
 *   vs_t  = V_t + D_t
 *   pg_t  = rho_t (r_t + gamma*boot'_t - V_t), boot'_t = vs_{t+1} while the
 *           episode goes on (vs_T = last value), bootstrap_values[t] at a
 *           truncation, 0 at a termination.
 */
int oracle_vtrace(const float *log_rhos, const float *rewards, const float *values,
                  const float *terminateds, const float *truncateds,
                  const float *bootstrap_values, const float *last_values, double *vs,
                  double *pg_advantages, int64_t E, int64_t T, double gamma,
                  double lambda_, double rho_bar, double c_bar)
{
    if (check_common(rewards, values, E, T) || (E > 0 && T > 0 && (log_rhos == NULL || vs == NULL || pg_advantages == NULL)))
        return ORACLE_EINVAL;
    if (truncateds != NULL && bootstrap_values == NULL)
        return ORACLE_EINVAL;
    for (int64_t e = 0; e < E; ++e) {
        const int64_t row = e * T;
        double d_next = 0.0;
        for (int64_t t = T - 1; t >= 0; --t) {
            const int64_t i = row + t;
            int cont, trn;
            step_status(terminateds, truncateds, i, &cont, &trn);
            double ratio = exp((double)log_rhos[i]);
            double rho = fmin(rho_bar, ratio);
            double c = lambda_ * fmin(c_bar, ratio);
            double next_v = (t + 1 < T) ? (double)values[i + 1] : last_value(last_values, e);
            double td = (double)rewards[i] + gamma * bootstrap(cont, trn, next_v, bootstrap_values, i)
                        - (double)values[i];
            double d = rho * td;
            if (cont)
                d += gamma * c * d_next;
            vs[i] = (double)values[i] + d;
            d_next = d;
            double next_vs = (t + 1 < T) ? vs[i + 1] : last_value(last_values, e);
            pg_advantages[i] = rho * ((double)rewards[i]
                                      + gamma * bootstrap(cont, trn, next_vs, bootstrap_values, i)
                                      - (double)values[i]);
        }
    }
    return ORACLE_OK;
}

/*
 * Retrace(lambda) (README "Kernels": "off-policy return estimate with
 * truncated IS ratios"; with-truncations paragraph: terminated and truncated
 * are both mandatory and the continuation value is folded into
 * next_q_values_all at every step; Munos et al. 2016, the Retrace operator
 * with c_s = lambda * min(c_bar, pi/mu)):
 *   V'_t = sum_a next_target_probs[t][a] * next_q_values_all[t][a]
 *          (A == 1 and no probabilities: V'_t = next_q_values_all[t][0])
 *   delta_t = r_t + gamma * (terminated_t ? 0 : V'_t) - q_t
 *   c_{t+1} = lambda * min(c_bar, exp(log_rho_{t+1}))           (t < T-1)
 *   Dq_t    = delta_t + gamma c_{t+1} Dq_{t+1} while the episode goes on,
 *   Dq_t    = delta_t at a flagged step or at t = T-1
 *   Q_ret_t = q_t + Dq_t
 */
int oracle_retrace(const float *rewards, const float *q_values,
                   const float *next_q_values_all, const float *next_target_probs,
                   const float *log_rhos, const float *terminateds, const float *truncateds,
                   double *q_ret, int64_t E, int64_t T, int64_t A, double gamma,
                   double lambda_, double c_bar)
{
    if (check_common(rewards, q_values, E, T))
        return ORACLE_EINVAL;
    if (A < 1 || (A > 1 && next_target_probs == NULL))
        return ORACLE_EINVAL;
    if (E > 0 && T > 0 && (next_q_values_all == NULL || log_rhos == NULL || q_ret == NULL))
        return ORACLE_EINVAL;
    for (int64_t e = 0; e < E; ++e) {
        const int64_t row = e * T;
        double dq_next = 0.0;
        for (int64_t t = T - 1; t >= 0; --t) {
            const int64_t i = row + t;
            int cont, trn;
            step_status(terminateds, truncateds, i, &cont, &trn);
            double v_next = 0.0;
            if (next_target_probs == NULL) {
                v_next = (double)next_q_values_all[i * A];
            } else {
                for (int64_t a = 0; a < A; ++a)
                    v_next += (double)next_target_probs[i * A + a] * (double)next_q_values_all[i * A + a];
            }
            double delta = (double)rewards[i] + gamma * (is_set(terminateds, i) ? 0.0 : v_next)
                           - (double)q_values[i];
            double dq = delta;
            if (cont && t + 1 < T) {
                double c_next = lambda_ * fmin(c_bar, exp((double)log_rhos[i + 1]));
                dq += gamma * c_next * dq_next;
            }
            q_ret[i] = (double)q_values[i] + dq;
            dq_next = dq;
        }
    }
    return ORACLE_OK;
}

/*
 * TD(lambda) returns (README "Kernels": "lambda-return targets mixing one-step
 * TD and Monte Carlo"; Sutton & Barto 2018, chapter 12, the lambda-return in
 * recursive form):
 *   G_t = r_t + gamma ((1-lambda) V_{t+1} + lambda G_{t+1})  while the episode goes on,
 *   G_t = r_t + gamma bootstrap_values[t]                   at a truncation,
 *   G_t = r_t                                               at a termination,
 * with V_T = G_T = last value.
 */
int oracle_lambda_returns(const float *rewards, const float *values, const float *terminateds,
                          const float *truncateds, const float *bootstrap_values,
                          const float *last_values, double *returns, int64_t E, int64_t T,
                          double gamma, double lambda_)
{
    if (check_common(rewards, values, E, T) || (E > 0 && T > 0 && returns == NULL))
        return ORACLE_EINVAL;
    if (truncateds != NULL && bootstrap_values == NULL)
        return ORACLE_EINVAL;
    for (int64_t e = 0; e < E; ++e) {
        const int64_t row = e * T;
        const double lv = last_value(last_values, e);
        double g_next = lv;
        for (int64_t t = T - 1; t >= 0; --t) {
            const int64_t i = row + t;
            int cont, trn;
            step_status(terminateds, truncateds, i, &cont, &trn);
            double next_v = (t + 1 < T) ? (double)values[i + 1] : lv;
            double g;
            if (cont)
                g = (double)rewards[i] + gamma * ((1.0 - lambda_) * next_v + lambda_ * g_next);
            else if (trn)
                g = (double)rewards[i] + gamma * (double)bootstrap_values[i];
            else
                g = (double)rewards[i];
            returns[i] = g;
            g_next = g;
        }
    }
    return ORACLE_OK;
}

/*
 * Discounted returns (README "Kernels": "discounted reward-to-go"):
 *   R_t = r_t + gamma R_{t+1}                while the episode goes on,
 *   R_t = r_t + gamma bootstrap_values[t]    at a truncation,
 *   R_t = r_t                                at a termination,
 * with R_T = last value.
 */
int oracle_discounted_returns(const float *rewards, const float *terminateds,
                              const float *truncateds, const float *bootstrap_values,
                              const float *last_values, double *returns, int64_t E,
                              int64_t T, double gamma)
{
    if (check_common(rewards, returns, E, T))
        return ORACLE_EINVAL;
    if (truncateds != NULL && bootstrap_values == NULL)
        return ORACLE_EINVAL;
    for (int64_t e = 0; e < E; ++e) {
        const int64_t row = e * T;
        double r_next = last_value(last_values, e);
        for (int64_t t = T - 1; t >= 0; --t) {
            const int64_t i = row + t;
            int cont, trn;
            step_status(terminateds, truncateds, i, &cont, &trn);
            double ret = (double)rewards[i];
            if (cont)
                ret += gamma * r_next;
            else if (trn)
                ret += gamma * (double)bootstrap_values[i];
            returns[i] = ret;
            r_next = ret;
        }
    }
    return ORACLE_OK;
}

/*
 * Eligibility traces (README "Kernels": accumulating forward traces
 * e[t] = x[t] + gamma*lambda*(1-d)*e[t-1]).  Default reading: the done that
 * ends an episode at t-1 resets the trace at t,
 *   e_t = x_t + gamma*lambda e_{t-1}   if t > 0 and d_{t-1} == 0,
 *   e_t = x_t                          otherwise;
 * with done_starts_episode != 0 the flag is read at t itself (d_t in place of
 * d_{t-1} above: t is the first step of a new episode).
 */
int oracle_eligibility_traces(const float *x, const float *dones, double *traces,
                              int64_t E, int64_t T, double gamma, double lambda_,
                              int done_starts_episode)
{
    if (check_common(x, traces, E, T))
        return ORACLE_EINVAL;
    for (int64_t e = 0; e < E; ++e) {
        const int64_t row = e * T;
        double prev = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            const int64_t i = row + t;
            double cur = (double)x[i];
            const int reset = done_starts_episode ? is_set(dones, i) : (t > 0 && is_set(dones, i - 1));
            if (t > 0 && !reset)
                cur += gamma * lambda_ * prev;
            traces[i] = cur;
            prev = cur;
        }
    }
    return ORACLE_OK;
}

/*
 * Episodic prefix sum, fp32 input (README "Kernels": "episodic cumulative sum
 * with done-mask resets"):
 *   y_t = x_t + y_{t-1}   if t > 0 and d_{t-1} == 0,   y_t = x_t otherwise;
 * with done_starts_episode != 0, d_t replaces d_{t-1}.
 */
int oracle_episodic_prefix_sum_f32(const float *x, const float *dones, double *out,
                                   int64_t E, int64_t T, int done_starts_episode)
{
    if (check_common(x, out, E, T))
        return ORACLE_EINVAL;
    for (int64_t e = 0; e < E; ++e) {
        const int64_t row = e * T;
        double prev = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            const int64_t i = row + t;
            double cur = (double)x[i];
            const int reset = done_starts_episode ? is_set(dones, i) : (t > 0 && is_set(dones, i - 1));
            if (t > 0 && !reset)
                cur += prev;
            out[i] = cur;
            prev = cur;
        }
    }
    return ORACLE_OK;
}

/*
 * Episodic prefix sum, int32 input: the same recurrence in two's-complement
 * int32 arithmetic (each step's sum is reduced modulo 2^32), so that a sum
 * that overflows wraps the way 32-bit integer addition does.
 */
int oracle_episodic_prefix_sum_i32(const int32_t *x, const float *dones, int32_t *out,
                                   int64_t E, int64_t T, int done_starts_episode)
{
    if (check_common(x, out, E, T))
        return ORACLE_EINVAL;
    for (int64_t e = 0; e < E; ++e) {
        const int64_t row = e * T;
        int64_t prev = 0;
        for (int64_t t = 0; t < T; ++t) {
            const int64_t i = row + t;
            int64_t cur = (int64_t)x[i];
            const int reset = done_starts_episode ? is_set(dones, i) : (t > 0 && is_set(dones, i - 1));
            if (t > 0 && !reset)
                cur += prev;
            /* reduce modulo 2^32 into [-2^31, 2^31) */
            uint32_t low = (uint32_t)((uint64_t)cur & 0xffffffffu);
            int64_t wrapped = (low >= 0x80000000u) ? (int64_t)low - 4294967296LL : (int64_t)low;
            out[i] = (int32_t)wrapped;
            prev = wrapped;
        }
    }
    return ORACLE_OK;
}
