/*
 * gla_oracle.c -- plain, slow, fp64 CPU oracle for GTR's Key-only gated linear
 * attention (GLA) token mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * Sources (all formulas on the first page were lost in extraction; the prose
 * around them survives and fixes the plain reading written out below):
 *   [GTR-art]  "端侧实时感知新标杆！通用线性骨干网络GTR开源" (shuwu5.cn/article/3124)
 *     - 方法详解 §1 "骨干架构：Key-only 门控递归与四向交替扫描":
 *         per head, a dk x dv state; value-side decay fixed to 1, key-side
 *         adaptive forget gate only:
 *             S_t = diag(alpha_t) S_{t-1} + k_t^T v_t,   o_t = q_t S_t,
 *             alpha_t = exp(g_t);
 *         the gate comes from a low-rank projection with a temperature:
 *             g_t = logsigmoid(x_t W_down W_up + b) / tau;
 *         the output is RMS-normalised and multiplied by a SiLU output gate:
 *             y_t = RMSNorm(o_t) * SiLU(z_t),  z_t = x_t W_g;
 *         one scan direction per block out of LR, RL, TB, BT, with the 2-D
 *         grid order restored right after the scan.
 *   [GTR-lst]  "GTR: Gated Token Recurrence for Efficient Dense Prediction"
 *     (m.montaan.com/papers/2609.26590), Abstract: gated linear attention with
 *     alternating spatial scan directions.
 *
 * Readings taken where the page is silent (each one is also listed in the
 * design notes of the repository):
 *   - no feature map and no 1/sqrt(dk) inside the operator;
 *   - the state includes token t when o_t is read (inclusive causality);
 *   - LR = row-major raster, RL = LR reversed, TB = column-major (down each
 *     column, columns left to right), BT = TB reversed; the output is stored
 *     back at the grid index the scan visited (grid order restored);
 *   - RMSNorm over the dv values of one (token, head), eps = 1e-5 by default,
 *     weight w[dv] shared by all heads;
 *   - logsigmoid(u) = min(u,0) - log1p(exp(-|u|)), the overflow-free form.
 *
 * Every function is a direct transcription of the definition: token by token,
 * head by head, in fp64, with no blocking, fusion or reordering.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Scan orders (GTR-art 方法详解 §1): sequence position s -> grid index. */
enum { OR_LR = 0, OR_RL = 1, OR_TB = 2, OR_BT = 3, OR_ROTATE_BATCH = 4 };

static long scan_to_grid(int dir, long s, long gh, long gw)
{
    long T = gh * gw;
    long r;
    switch (dir) {
    case OR_LR: return s;
    case OR_RL: return T - 1 - s;
    case OR_TB: return (s % gh) * gw + s / gh;
    case OR_BT: r = T - 1 - s; return (r % gh) * gw + r / gh;
    default: return -1;
    }
}

static int dir_of_batch(int dir, int b) { return dir == OR_ROTATE_BATCH ? (b % 4) : dir; }

int oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* The grid index visited at scan position s (exported so tests can check the
 * maps against explicit grid flips and transposes). */
long oracle_scan_index(int dir, long s, long gh, long gw) { return scan_to_grid(dir, s, gh, gw); }

/*
 * Gate projection, GTR-art 方法详解 §1 (rank-r projection with temperature tau):
 *   g[n, j] = logsigmoid( sum_r (sum_c x[n,c] w_down[c,r]) w_up[r,j] + bias[j] ) / tau
 * x: [N, d_model], w_down: [d_model, rank], w_up: [rank, HD], bias: [HD] or NULL,
 * g: [N, HD].  All row-major fp64.
 */
int oracle_gate_f64(const double *x, const double *w_down, const double *w_up,
                    const double *bias, double *g, long N, int d_model, int rank,
                    int HD, double tau)
{
    if (!x || !w_down || !w_up || !g || N < 0 || d_model <= 0 || rank <= 0 || HD <= 0 || !(tau > 0))
        return -1;
    if (rank > 256) return -2;
    long n;
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n) {
        double low[256];
        int r, c, j;
        const double *xr = x + n * (long)d_model;
        for (r = 0; r < rank; ++r) {
            double acc = 0.0;
            for (c = 0; c < d_model; ++c) acc += xr[c] * w_down[(long)c * rank + r];
            low[r] = acc;
        }
        for (j = 0; j < HD; ++j) {
            double u = bias ? bias[j] : 0.0;
            for (r = 0; r < rank; ++r) u += low[r] * w_up[(long)r * HD + j];
            double ls = (u < 0.0 ? u : 0.0) - log1p(exp(-fabs(u)));
            g[n * (long)HD + j] = ls / tau;
        }
    }
    return 0;
}

/*
 * The Key-only GLA forward, GTR-art 方法详解 §1, one head at a time, token by
 * token in scan order:
 *   S = 0
 *   for s in 0..T-1:  t = pi_dir(s)
 *     S[i][j] = exp(g[t,i]) * S[i][j] + k[t,i] * v[t,j]
 *     o[j]    = sum_i q[t,i] * S[i][j]
 *     y[t,j]  = o[j] / sqrt(mean_j o[j]^2 + eps) * w[j] * z[t,j] * sigmoid(z[t,j])
 * Layouts: q,k,g: [B, T, H, dk]; v,z,y,o_raw: [B, T, H, dv]; w: [dv] or NULL
 * (all ones); T = gh*gw with grid index t = row*gw + col.  o_raw (nullable)
 * receives o before the normalisation.  dir in {LR,RL,TB,BT,ROTATE_BATCH};
 * ROTATE_BATCH uses direction (b mod 4) for batch entry b.
 */
int oracle_gla_fwd_f64(const double *q, const double *k, const double *v, const double *g,
                       const double *z, const double *w, double *y, double *o_raw,
                       int B, int H, int gh, int gw, int dk, int dv, int dir, double eps)
{
    if (!q || !k || !v || !g || !z || !y || B < 0 || H <= 0 || gh <= 0 || gw <= 0 ||
        dk <= 0 || dv <= 0 || dir < 0 || dir > 4 || eps < 0)
        return -1;
    long T = (long)gh * gw;
    long bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < (long)B * H; ++bh) {
        int b = (int)(bh / H), h = (int)(bh % H);
        int d = dir_of_batch(dir, b);
        double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
        double *o = (double *)malloc((size_t)dv * sizeof(double));
        long s;
        for (s = 0; s < T; ++s) {
            long t = scan_to_grid(d, s, gh, gw);
            long rowk = ((long)b * T + t) * H + h;
            const double *qt = q + rowk * dk, *kt = k + rowk * dk, *gt = g + rowk * dk;
            const double *vt = v + rowk * dv, *zt = z + rowk * dv;
            int i, j;
            for (i = 0; i < dk; ++i) {
                double a = exp(gt[i]);
                double *Si = S + (long)i * dv;
                for (j = 0; j < dv; ++j) Si[j] = a * Si[j] + kt[i] * vt[j];
            }
            double ss = 0.0;
            for (j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (i = 0; i < dk; ++i) acc += qt[i] * S[(long)i * dv + j];
                o[j] = acc;
                ss += acc * acc;
            }
            double inv = 1.0 / sqrt(ss / dv + eps);
            for (j = 0; j < dv; ++j) {
                double silu = zt[j] / (1.0 + exp(-zt[j]));
                double wj = w ? w[j] : 1.0;
                y[rowk * dv + j] = o[j] * inv * wj * silu;
                if (o_raw) o_raw[rowk * dv + j] = o[j];
            }
        }
        free(S);
        free(o);
    }
    return 0;
}

/*
 * The state after the last token of every chunk of `chunk` scan positions
 * (GTR-art 方法详解 §4 "硬件感知分块推理算子": the chunk-boundary states the
 * light sequential pass carries).  states: [B, H, ceil(T/chunk), dk, dv];
 * entry c holds S after scan position min((c+1)*chunk, T) - 1, i.e. the state
 * a chunk c+1 starts from.
 */
int oracle_gla_chunk_states_f64(const double *k, const double *v, const double *g, double *states,
                                int B, int H, int gh, int gw, int dk, int dv, int dir, int chunk)
{
    if (!k || !v || !g || !states || B < 0 || H <= 0 || gh <= 0 || gw <= 0 || dk <= 0 ||
        dv <= 0 || dir < 0 || dir > 4 || chunk <= 0)
        return -1;
    long T = (long)gh * gw;
    long Nc = (T + chunk - 1) / chunk;
    long bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < (long)B * H; ++bh) {
        int b = (int)(bh / H), h = (int)(bh % H);
        int d = dir_of_batch(dir, b);
        double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
        long s;
        for (s = 0; s < T; ++s) {
            long t = scan_to_grid(d, s, gh, gw);
            long rowk = ((long)b * T + t) * H + h;
            const double *kt = k + rowk * dk, *gt = g + rowk * dk, *vt = v + rowk * dv;
            int i, j;
            for (i = 0; i < dk; ++i) {
                double a = exp(gt[i]);
                for (j = 0; j < dv; ++j) S[(long)i * dv + j] = a * S[(long)i * dv + j] + kt[i] * vt[j];
            }
            if ((s + 1) % chunk == 0 || s == T - 1) {
                long c = s / chunk;
                memcpy(states + ((bh * Nc) + c) * (long)dk * dv, S, (size_t)dk * dv * sizeof(double));
            }
        }
        free(S);
    }
    return 0;
}
