/*
 * m2_oracle.c -- plain, slow CPU oracle for the Mamba-2 recurrent-state path.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark load this library. The product path never calls it,
 * and it shares no code, header, table or helper with the CUDA path.
 *
 * Everything is computed in IEEE double precision with the C library's exp,
 * log1p and nearbyint. Loops follow the definitions in the order they are
 * stated; sums over the state dimension run in ascending n. There is no
 * blocking, fusion or reordering. Threading, if any, is the caller's business
 * across independent sequences.
 *
 * The operations (names as on the vllm.cpp issue page "NemotronH runs the
 * PREFILL mamba kernels at decode", section "The divergence"):
 *
 *   causal_conv1d_update -- a depthwise causal convolution of width K over the
 *     xBC channels, fed by a rolling cache of the last K-1 raw inputs of each
 *     channel, read and written in place at the sequence's slot;
 *   selective_state_update -- one step of the Mamba-2 recurrence per head h:
 *       dt  = softplus(dt_raw[h] + dt_bias[h])
 *       A   = -exp(A_log[h])
 *       dA  = exp(dt * A)
 *       S'[h,p,n] = S[h,p,n] * dA + (dt * x[h,p]) * B[g(h),n]
 *       y[h,p]    = sum_n S'[h,p,n] * C[g(h),n] + D[h] * x[h,p]
 *       y[h,p]   *= silu(z[h,p])            (when z is given)
 *     with heads mapped to groups by g(h) = h / (H/G) (the issue's "hpg = H/G",
 *     section "Confirm or refute").
 *   chunked prefill scan -- must land on the same state as T sequential
 *     selective_state_update steps; the definition used here is exactly that
 *     loop, with the working state kept unrounded across the T tokens.
 *   gated RMSNorm -- the mixer's `norm` tensor (Nemotron-H-8B-Base-8K model
 *     record, the tensor list of the Mamba-2 mixer layers): the gated y is
 *     normalised by its root mean square over groups of H*P/G consecutive
 *     channels and scaled by the norm weight.
 *
 * Shapes follow the Nemotron-H-8B-Base-8K model record (ssm_state_size N,
 * mamba_head_dim P, mamba_num_heads H, n_groups G): the state of one sequence
 * is [H][P][N], N fastest; xBC is [x: H*P | B: G*N | C: G*N].
 *
 * Compile-time switches M2O_MUTANT_* plant one deliberate mistake each; they
 * exist only so the tests can show that the oracle's pins catch such mistakes.
 * The default build defines none of them.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define M2O_ROUND_F32 0
#define M2O_ROUND_BF16 1
#define M2O_ROUND_NONE 2
#define M2O_ROUND_F16 3

/* ---------------------------------------------------------------- rounding */

/* Round to the nearest float32 (ties to even): the C conversion rounds in the
 * current mode, which is round-to-nearest-even by default. */
double m2o_round_f32(double x) { return (double)(float)x; }

/* Round to the nearest bfloat16 (8-bit significand, float32 exponent range),
 * ties to even, straight from double: the value is scaled by its own ulp so
 * that nearbyint does the rounding in one step. Non-finite inputs pass
 * through; overflow gives an infinity. */
double m2o_round_bf16(double x) {
    if (!isfinite(x) || x == 0.0) return x;
    int e;
    frexp(x, &e);                   /* |x| in [2^(e-1), 2^e) */
    int ulp_exp = (e - 1) - 7;      /* 7 fraction bits after the leading one */
    if (ulp_exp < -133) ulp_exp = -133; /* bfloat16 subnormal spacing 2^-133 */
    double q = ldexp(x, -ulp_exp);
#ifdef M2O_MUTANT_BF16_TRUNC
    double r = ldexp(trunc(q), ulp_exp);
#else
    double r = ldexp(nearbyint(q), ulp_exp);
#endif
    if (fabs(r) > 3.3895313892515355e38) r = copysign(INFINITY, x);
    return r;
}

/* Round to the nearest IEEE binary16 (11-bit significand, exponents -14..15,
 * subnormal spacing 2^-24), ties to even, straight from double; beyond the
 * largest finite value (65504) the result is an infinity. */
double m2o_round_f16(double x) {
    if (!isfinite(x) || x == 0.0) return x;
    int e;
    frexp(x, &e);
    int ulp_exp = (e - 1) - 10;
    if (ulp_exp < -24) ulp_exp = -24;
    double r = ldexp(nearbyint(ldexp(x, -ulp_exp)), ulp_exp);
    if (fabs(r) > 65504.0) r = copysign(INFINITY, x);
    return r;
}

double m2o_round(double x, int mode) {
    if (mode == M2O_ROUND_F32) return m2o_round_f32(x);
    if (mode == M2O_ROUND_BF16) return m2o_round_bf16(x);
    if (mode == M2O_ROUND_F16) return m2o_round_f16(x);
    return x;
}

/* Round every element of x in place (used where a value is stored in a
 * narrower precision between two operations). */
void m2o_round_array(double* x, int64_t n, int mode) {
    for (int64_t i = 0; i < n; ++i) x[i] = m2o_round(x[i], mode);
}

/* ------------------------------------------------------------- activations */

/* softplus(v) = log(1 + exp(v)), taken as v itself above 20 (where the two
 * agree to double precision in every digit that matters to the result). */
double m2o_softplus(double v) {
    if (v > 20.0) return v;
    return log1p(exp(v));
}

/* silu(v) = v * sigmoid(v) = v / (1 + exp(-v)). */
double m2o_silu(double v) { return v / (1.0 + exp(-v)); }

/* The gate applied to y: silu(z). */
static double gate(double zv) {
#ifdef M2O_MUTANT_GATE_SIGMOID
    return 1.0 / (1.0 + exp(-zv));
#else
    return m2o_silu(zv);
#endif
}

/* --------------------------------------------------- causal_conv1d_update */

/*
 * Depthwise causal convolution over T tokens of one sequence.
 *
 *   conv_state [K-1][C]  in/out: raw inputs of the previous K-1 tokens, oldest
 *                        row first; on return it holds the last K-1 raw inputs
 *                        of the window (an exact copy, no arithmetic).
 *   x_raw      [T][C]    raw xBC rows.
 *   w          [C][K]    tap k multiplies the input k steps after the oldest in
 *                        the window, so w[c][K-1] multiplies the newest input.
 *   bias       [C]       or NULL.
 *   activation           0 = none, 1 = SiLU after the bias.
 *   out        [T][C]    post-conv values (double, no rounding).
 *
 * For token t the window is (oldest .. newest) = the K-1 inputs before t, then
 * x_raw[t]; out[t][c] = bias[c] + sum_k w[c][k] * window[k].
 */
void m2o_conv1d(int C, int K, int T, double* conv_state, const double* x_raw,
                const double* w, const double* bias, int activation, double* out) {
    double window[16];
    for (int c = 0; c < C; ++c) {
        for (int k = 0; k < K - 1; ++k) window[k] = conv_state[(size_t)k * C + c];
        for (int t = 0; t < T; ++t) {
            window[K - 1] = x_raw[(size_t)t * C + c];
            double acc = bias ? bias[c] : 0.0;
            for (int k = 0; k < K; ++k) {
#ifdef M2O_MUTANT_CONV_FLIP
                acc += w[(size_t)c * K + (K - 1 - k)] * window[k];
#else
                acc += w[(size_t)c * K + k] * window[k];
#endif
            }
            out[(size_t)t * C + c] = activation ? m2o_silu(acc) : acc;
            for (int k = 0; k < K - 1; ++k) window[k] = window[k + 1];
        }
#ifndef M2O_MUTANT_NO_ROLL
        for (int k = 0; k < K - 1; ++k) conv_state[(size_t)k * C + c] = window[k];
#endif
    }
}

/* ------------------------------------------------- selective_state_update */

/*
 * One recurrence step for one sequence, all heads, on a double working state.
 *
 *   state  [H][P][N]  in/out, not rounded here.
 *   xbc    [H*P + 2*G*N]  post-conv x | B | C.
 *   dt_raw [H], dt_bias [H], A_log [H], D [H].
 *   z      [H*P] or NULL.
 *   y      [H*P] out.
 */
static void ssm_step_unrounded(int H, int P, int N, int G, double* state, const double* xbc,
                               const double* dt_raw, const double* dt_bias, const double* A_log,
                               const double* D, const double* z, double* y) {
    const int hpg = H / G;
    const double* x = xbc;
#ifdef M2O_MUTANT_SWAP_BC
    const double* Cm = xbc + (size_t)H * P;
    const double* Bm = Cm + (size_t)G * N;
#else
    const double* Bm = xbc + (size_t)H * P;
    const double* Cm = Bm + (size_t)G * N;
#endif
    for (int h = 0; h < H; ++h) {
#ifdef M2O_MUTANT_GROUP_MOD
        const int g = h % G;
#else
        const int g = h / hpg;
#endif
#ifdef M2O_MUTANT_DT_NO_BIAS
        const double dt = m2o_softplus(dt_raw[h]);
#else
        const double dt = m2o_softplus(dt_raw[h] + dt_bias[h]);
#endif
#ifdef M2O_MUTANT_A_SIGN
        const double A = exp(A_log[h]);
#else
        const double A = -exp(A_log[h]);
#endif
        const double dA = exp(dt * A);
        const double* Bg = Bm + (size_t)g * N;
        const double* Cg = Cm + (size_t)g * N;
        for (int p = 0; p < P; ++p) {
            double* s = state + ((size_t)h * P + p) * N;
            const double xv = x[(size_t)h * P + p];
            double acc = 0.0;
            for (int n = 0; n < N; ++n) {
                const double s_old = s[n];
#ifdef M2O_MUTANT_DROP_DT_INPUT
                const double s_new = s_old * dA + xv * Bg[n];
#else
                const double s_new = s_old * dA + (dt * xv) * Bg[n];
#endif
                s[n] = s_new;
#ifdef M2O_MUTANT_Y_OLD_STATE
                acc += s_old * Cg[n];
#elif defined(M2O_MUTANT_Y_USES_B)
                acc += s_new * Bg[n];
#else
                acc += s_new * Cg[n];
#endif
            }
#ifdef M2O_MUTANT_DROP_D
            double yv = acc;
#else
            double yv = acc + D[h] * xv;
#endif
            if (z) yv *= gate(z[(size_t)h * P + p]);
            y[(size_t)h * P + p] = yv;
        }
    }
}

/*
 * One decode step as stored in a cache: the state is read from its storage
 * precision (already exact in double), updated, and rounded back to it
 * (round_mode: 0 = float32, 1 = bfloat16, 2 = keep double). y is computed
 * from the unrounded new state.
 */
void m2o_ssm_step(int H, int P, int N, int G, double* state, int round_mode, const double* xbc,
                  const double* dt_raw, const double* dt_bias, const double* A_log,
                  const double* D, const double* z, double* y) {
    ssm_step_unrounded(H, P, N, G, state, xbc, dt_raw, dt_bias, A_log, D, z, y);
    const size_t n = (size_t)H * P * N;
    for (size_t i = 0; i < n; ++i) state[i] = m2o_round(state[i], round_mode);
}

/*
 * T tokens of one sequence, the definition of the chunked prefill scan: T
 * sequential steps with the working state in double throughout, rounded once
 * to round_mode at the end.
 *
 *   xbc [T][H*P + 2*G*N], dt_raw [T][H], z [T][H*P] or NULL, y [T][H*P].
 */
void m2o_ssm_scan(int H, int P, int N, int G, int T, double* state, int round_mode,
                  const double* xbc, const double* dt_raw, const double* dt_bias,
                  const double* A_log, const double* D, const double* z, double* y) {
    const size_t cd = (size_t)H * P + 2 * (size_t)G * N;
    const size_t hp = (size_t)H * P;
    for (int t = 0; t < T; ++t) {
        ssm_step_unrounded(H, P, N, G, state, xbc + t * cd, dt_raw + (size_t)t * H, dt_bias,
                           A_log, D, z ? z + t * hp : NULL, y + t * hp);
    }
    const size_t n = (size_t)H * P * N;
    for (size_t i = 0; i < n; ++i) state[i] = m2o_round(state[i], round_mode);
}

/*
 * Gated RMSNorm of one row of mixer output. v is the gated y (y * silu(z), as
 * m2o_ssm_step returns it: the gate comes before the norm); the HP channels
 * split into G groups of L = HP/G consecutive channels, and in each group
 *     ms     = (1/L) * sum_c v[c]^2
 *     out[c] = v[c] / sqrt(ms + eps) * w[c]
 */
void m2o_group_rmsnorm(int HP, int G, double eps, const double* v, const double* w, double* out) {
#ifdef M2O_MUTANT_NORM_WHOLE_ROW
    G = 1;
#endif
    const int L = HP / G;
    for (int gi = 0; gi < G; ++gi) {
        const double* vg = v + (size_t)gi * L;
        double ss = 0.0;
        for (int c = 0; c < L; ++c) ss += vg[c] * vg[c];
        const double ms = ss / L;
#ifdef M2O_MUTANT_NORM_EPS_OUTSIDE
        const double denom = sqrt(ms) + eps;
#else
        const double denom = sqrt(ms + eps);
#endif
        for (int c = 0; c < L; ++c) {
            const size_t i = (size_t)gi * L + c;
#ifdef M2O_MUTANT_NORM_NO_WEIGHT
            out[i] = v[i] / denom;
#else
            out[i] = v[i] / denom * w[i];
#endif
        }
    }
}

/* Version tag so the Python side can tell a mutant build from the default. */
const char* m2o_build_tag(void) {
#if defined(M2O_MUTANT_CONV_FLIP)
    return "mutant:conv_flip";
#elif defined(M2O_MUTANT_GROUP_MOD)
    return "mutant:group_mod";
#elif defined(M2O_MUTANT_A_SIGN)
    return "mutant:a_sign";
#elif defined(M2O_MUTANT_DROP_DT_INPUT)
    return "mutant:drop_dt_input";
#elif defined(M2O_MUTANT_Y_OLD_STATE)
    return "mutant:y_old_state";
#elif defined(M2O_MUTANT_Y_USES_B)
    return "mutant:y_uses_b";
#elif defined(M2O_MUTANT_DROP_D)
    return "mutant:drop_d";
#elif defined(M2O_MUTANT_BF16_TRUNC)
    return "mutant:bf16_trunc";
#elif defined(M2O_MUTANT_GATE_SIGMOID)
    return "mutant:gate_sigmoid";
#elif defined(M2O_MUTANT_NO_ROLL)
    return "mutant:no_roll";
#elif defined(M2O_MUTANT_SWAP_BC)
    return "mutant:swap_bc";
#elif defined(M2O_MUTANT_DT_NO_BIAS)
    return "mutant:dt_no_bias";
#elif defined(M2O_MUTANT_NORM_WHOLE_ROW)
    return "mutant:norm_whole_row";
#elif defined(M2O_MUTANT_NORM_EPS_OUTSIDE)
    return "mutant:norm_eps_outside";
#elif defined(M2O_MUTANT_NORM_NO_WEIGHT)
    return "mutant:norm_no_weight";
#else
    return "oracle";
#endif
}
