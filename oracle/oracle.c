/*
 * Plain fp64 CPU oracle for the activation-sparse gated FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the package's smoke check and the bench's
 * CPU-baseline leg use it.  It shares no code, header or table with the CUDA
 * library: it is written from the method's definition, slowly and plainly.
 *
 * Source: "Sparser, Faster, Lighter Transformer Language Models" (Cetin et
 * al., ICML 2026), as summarised on the pwwt.cn page:
 *   - section 01, figure "Gated FFN up, gate and down projection": the gated
 *     FFN y = (ReLU(x W_gate) (.) (x W_up)) W_down, with ReLU as the gate
 *     activation giving exact zeros (the formula itself is lost from the
 *     page; the plain reading with no bias terms is used);
 *   - section 02, figures "TwELL cuts the column direction into tiles" and
 *     "gate projection with TwELL storage generation": TwELL keeps, per row
 *     and per 1-D column tile of width T, a count, the nonzero values and
 *     their local column indices;
 *   - section 02 (last paragraph): up and down projections done in one pass
 *     without materialising h;
 *   - section 03, figure "routing of the hybrid-format sparse operator": rows
 *     with few nonzeros go to a compact ELL matrix, heavy rows to a dense
 *     backup path; the kongchang.com page ("custom CUDA kernels: fusion and
 *     compression") adds that TwELL is compressed into this hybrid form.
 * The backward formulas are not printed on the pages; they are the plain
 * derivatives of the gated FFN above.
 *
 * Value rounding: stored activations are rounded to the storage dtype with
 * round-to-nearest-even (kind 0 = keep fp64, 1 = fp32, 2 = bf16, 3 = fp16).
 * The activity test is g > 0 (NaN and -0 are inactive).
 *
 * Layouts (row-major, contiguous):
 *   x [N][d]; wg_t, wu_t, wd [F][d] (row j = column j of W_gate / W_up,
 *   row j of W_down); g [N][F];
 *   TwELL: count [N][F/T] (true count), idx [N][F/T][C] (local column,
 *   ascending), val [N][F/T][C]; only the first min(count, C) slots of a
 *   tile are meaningful.
 *   Hybrid: row_nnz [N], spill_slot [N] (-1 for ELL rows), spill_rows
 *   [S_max], ell_idx [N][K] (global column), ell_a / ell_u [N][K],
 *   spill_a / spill_u [S_max][F].
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ---------------------------------------------------------------- rounding */

/* Round-to-nearest-even of v to a binary format with p significant bits,
 * smallest spacing 2^qmin (subnormals) and largest finite value maxv. */
static double round_format(double v, int p, int qmin, double maxv) {
    if (v == 0.0 || !isfinite(v)) return v;
    int e;
    frexp(v, &e);                 /* v = m 2^e, 1/2 <= |m| < 1: spacing 2^(e-p) */
    int q = e - p;
    if (q < qmin) q = qmin;
    double r = nearbyint(ldexp(v, -q));   /* default mode: nearest, ties even */
    double out = ldexp(r, q);
    if (fabs(out) > maxv) out = copysign(INFINITY, v);
    return out;
}

double oracle_round_value(double v, int kind) {
    switch (kind) {
    case 1: return round_format(v, 24, -149, ldexp(2.0 - ldexp(1.0, -23), 127));
    case 2: return round_format(v, 8, -133, ldexp(2.0 - ldexp(1.0, -7), 127));
    case 3: return round_format(v, 11, -24, 65504.0);
    default: return v;
    }
}

void oracle_round_array(const double* v, int64_t n, int kind, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_round_value(v[i], kind);
}

/* ----------------------------------------------------- gate pre-activation */

/* g[t][j] = sum_i x[t][i] * W_gate[i][j]   (W_gate[i][j] = wg_t[j][i]) */
void oracle_gate_preact(const double* x, const double* wg_t, int64_t n, int64_t d,
                        int64_t f, double* g) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t) {
        const double* xt = x + t * d;
        for (int64_t j = 0; j < f; ++j) {
            const double* w = wg_t + j * d;
            double s = 0.0;
            for (int64_t i = 0; i < d; ++i) s += xt[i] * w[i];
            g[t * f + j] = s;
        }
    }
}

/* ------------------------------------------------------------- TwELL pack */

/* For every row t and tile b (columns bT .. bT+T-1), scan the tile in
 * ascending column order; a column is active iff g > 0.  The first C active
 * columns are kept as (local index, ReLU(g) rounded to the value dtype);
 * count holds the true number of active columns, which may exceed C.
 * Returns the number of tiles whose count exceeds C. */
int64_t oracle_twell_pack(const double* g, int64_t n, int64_t f, int tile, int cap,
                          int val_kind, uint8_t* count, uint8_t* idx, double* val) {
    const int64_t nt = f / tile;
    int64_t overflow = 0;
    for (int64_t t = 0; t < n; ++t) {
        for (int64_t b = 0; b < nt; ++b) {
            const int64_t seg = t * nt + b;
            int c = 0;
            for (int jj = 0; jj < tile; ++jj) {
                const double v = g[t * f + b * tile + jj];
                if (v > 0.0) {
                    if (c < cap) {
                        idx[seg * cap + c] = (uint8_t)jj;
                        val[seg * cap + c] = oracle_round_value(v, val_kind);
                    }
                    ++c;
                }
            }
            count[seg] = (uint8_t)c;
            if (c > cap) ++overflow;
        }
    }
    return overflow;
}

/* Dense [N][F] matrix holding the stored TwELL entries, zero elsewhere. */
void oracle_twell_unpack(const uint8_t* count, const uint8_t* idx, const double* val,
                         int64_t n, int64_t f, int tile, int cap, double* h) {
    const int64_t nt = f / tile;
    memset(h, 0, sizeof(double) * (size_t)(n * f));
    for (int64_t t = 0; t < n; ++t)
        for (int64_t b = 0; b < nt; ++b) {
            const int64_t seg = t * nt + b;
            const int c = count[seg] < cap ? count[seg] : cap;
            for (int s = 0; s < c; ++s)
                h[t * f + b * tile + idx[seg * cap + s]] = val[seg * cap + s];
        }
}

/* ------------------------------------------------------ fused up and down */

/* y[t] = sum over stored entries (j, a) of row t of  a * (x[t] . W_up[:, j]) * W_down[j, :]
 * (h_j = a * u_j is formed and used at once, never stored). */
void oracle_fused_up_down(const double* x, const uint8_t* count, const uint8_t* idx,
                          const double* val, const double* wu_t, const double* wd,
                          int64_t n, int64_t d, int64_t f, int tile, int cap, double* y) {
    const int64_t nt = f / tile;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < n; ++t) {
        const double* xt = x + t * d;
        double* yt = y + t * d;
        for (int64_t i = 0; i < d; ++i) yt[i] = 0.0;
        for (int64_t b = 0; b < nt; ++b) {
            const int64_t seg = t * nt + b;
            const int c = count[seg] < cap ? count[seg] : cap;
            for (int s = 0; s < c; ++s) {
                const int64_t j = b * tile + idx[seg * cap + s];
                const double* wu = wu_t + j * d;
                double u = 0.0;
                for (int64_t i = 0; i < d; ++i) u += xt[i] * wu[i];
                const double h = val[seg * cap + s] * u;
                const double* w = wd + j * d;
                for (int64_t i = 0; i < d; ++i) yt[i] += h * w[i];
            }
        }
    }
}

/* ------------------------------------------------------------ dense FFN */

/* y = (ReLU(x W_gate) (.) (x W_up)) W_down by the definition, column j of the
 * hidden layer at a time in ascending order. */
void oracle_dense_ffn(const double* x, const double* wg_t, const double* wu_t,
                      const double* wd, int64_t n, int64_t d, int64_t f, double* y) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < n; ++t) {
        const double* xt = x + t * d;
        double* yt = y + t * d;
        for (int64_t i = 0; i < d; ++i) yt[i] = 0.0;
        for (int64_t j = 0; j < f; ++j) {
            double g = 0.0, u = 0.0;
            for (int64_t i = 0; i < d; ++i) {
                g += xt[i] * wg_t[j * d + i];
                u += xt[i] * wu_t[j * d + i];
            }
            const double h = (g > 0.0 ? g : 0.0) * u;
            for (int64_t i = 0; i < d; ++i) yt[i] += h * wd[j * d + i];
        }
    }
}

/* ------------------------------------------------------------ hybrid pack */

/* Compress TwELL into the hybrid form.  Row t's nonzero count is the number
 * of stored entries, sum over tiles of min(count, C); a row with a tile whose
 * count exceeds C has lost entries to the capacity and cannot be an exact ELL
 * row, so if its stored count is <= K it is set to K + 1 and the row goes to
 * the spill (the dense backup path, where a forward given W_gate recomputes
 * it: the pages' dense path for the rows that do not fit the compact
 * format).  Rows with count <= K are ELL rows: their entries, in ascending global column, fill
 * ell_idx / ell_a [t][0 .. count) (the rest of the row is -1 / 0).  Rows with
 * count > K are spill rows, numbered in ascending t; the first S_max of them
 * get a dense row of spill_a (zero where inactive) and spill_slot[t] = rank;
 * rows ranked S_max or later are dropped (spill_slot -1, counted in the
 * return value's high half).  Returns n_spill | (dropped << 32). */
int64_t oracle_hybrid_pack(const uint8_t* count, const uint8_t* idx, const double* val,
                           int64_t n, int64_t f, int tile, int cap, int k, int s_max,
                           int32_t* row_nnz, int32_t* spill_slot, int32_t* spill_rows,
                           int32_t* ell_idx, double* ell_a, double* spill_a) {
    const int64_t nt = f / tile;
    int64_t n_spill = 0, dropped = 0;
    for (int64_t t = 0; t < n; ++t) {
        int64_t nnz = 0;
        int over = 0;
        for (int64_t b = 0; b < nt; ++b) {
            const int c = count[t * nt + b];
            nnz += c < cap ? c : cap;
            if (c > cap) over = 1;
        }
        if (over && nnz <= k) nnz = k + 1;
        row_nnz[t] = (int32_t)nnz;
        for (int s = 0; s < k; ++s) { ell_idx[t * k + s] = -1; ell_a[t * k + s] = 0.0; }
        if (nnz <= k) {
            spill_slot[t] = -1;
            int64_t w = 0;
            for (int64_t b = 0; b < nt; ++b) {
                const int64_t seg = t * nt + b;
                const int c = count[seg] < cap ? count[seg] : cap;
                for (int s = 0; s < c; ++s, ++w) {
                    ell_idx[t * k + w] = (int32_t)(b * tile + idx[seg * cap + s]);
                    ell_a[t * k + w] = val[seg * cap + s];
                }
            }
        } else {
            if (n_spill < s_max) {
                spill_slot[t] = (int32_t)n_spill;
                spill_rows[n_spill] = (int32_t)t;
                double* row = spill_a + n_spill * f;
                for (int64_t j = 0; j < f; ++j) row[j] = 0.0;
                for (int64_t b = 0; b < nt; ++b) {
                    const int64_t seg = t * nt + b;
                    const int c = count[seg] < cap ? count[seg] : cap;
                    for (int s = 0; s < c; ++s) row[b * tile + idx[seg * cap + s]] = val[seg * cap + s];
                }
            } else {
                spill_slot[t] = -1;
                ++dropped;
            }
            ++n_spill;
        }
    }
    return n_spill | (dropped << 32);
}

/* ------------------------------------------------------ hybrid forward */

/* ELL rows: y[t] = sum_s a * u * W_down[j] with u = x[t] . W_up[:, j], and u
 * is saved in ell_u.  Spill rows: the dense row U = x[t] W_up is saved in
 * spill_u and y[t] = (A (.) U) W_down.  Dropped rows get y = 0. */
void oracle_hybrid_fwd(const double* x, const int32_t* row_nnz, const int32_t* spill_slot,
                       const int32_t* ell_idx, const double* ell_a, const double* spill_a,
                       const double* wu_t, const double* wd, int64_t n, int64_t d, int64_t f,
                       int k, double* ell_u, double* spill_u, double* y) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < n; ++t) {
        const double* xt = x + t * d;
        double* yt = y + t * d;
        for (int64_t i = 0; i < d; ++i) yt[i] = 0.0;
        if (row_nnz[t] <= k) {
            for (int s = 0; s < k; ++s) ell_u[t * k + s] = 0.0;
            for (int s = 0; s < row_nnz[t]; ++s) {
                const int64_t j = ell_idx[t * k + s];
                double u = 0.0;
                for (int64_t i = 0; i < d; ++i) u += xt[i] * wu_t[j * d + i];
                ell_u[t * k + s] = u;
                const double h = ell_a[t * k + s] * u;
                for (int64_t i = 0; i < d; ++i) yt[i] += h * wd[j * d + i];
            }
        } else if (spill_slot[t] >= 0) {
            const int64_t r = spill_slot[t];
            for (int64_t j = 0; j < f; ++j) {
                double u = 0.0;
                for (int64_t i = 0; i < d; ++i) u += xt[i] * wu_t[j * d + i];
                spill_u[r * f + j] = u;
                const double h = spill_a[r * f + j] * u;
                for (int64_t i = 0; i < d; ++i) yt[i] += h * wd[j * d + i];
            }
        }
    }
}

/* ----------------------------------------------------- hybrid backward */

/* Gradients of y = sum_j a_j u_j W_down[j] with a_j = ReLU(g_j),
 * u_j = x . W_up[:, j], g_j = x . W_gate[:, j], over the active entries kept
 * in the hybrid form (a_j > 0 there, so ReLU'(g_j) = 1):
 *   dh_j = dy . W_down[j]      du_j = dh_j a_j      dg_j = dh_j u_j
 *   dx   = sum_j du_j W_up[:, j] + dg_j W_gate[:, j]
 *   dW_down[j] = sum_t a_tj u_tj dy_t
 *   dW_up[:, j] = sum_t du_tj x_t        dW_gate[:, j] = sum_t dg_tj x_t
 * Entries absent from the hybrid form (inactive or dropped) contribute 0.
 * dwg_t / dwu_t are stored neuron-major like the weights ([F][d]). */
void oracle_hybrid_bwd(const double* x, const double* dy, const int32_t* row_nnz,
                       const int32_t* spill_slot, const int32_t* ell_idx,
                       const double* ell_a, const double* ell_u, const double* spill_a,
                       const double* spill_u, const double* wg_t, const double* wu_t,
                       const double* wd, int64_t n, int64_t d, int64_t f, int k,
                       double* dx, double* dwg_t, double* dwu_t, double* dwd,
                       double* du_scratch, double* dg_scratch) {
    /* du, dg as dense [N][F] scratch (zero where no entry) */
    memset(du_scratch, 0, sizeof(double) * (size_t)(n * f));
    memset(dg_scratch, 0, sizeof(double) * (size_t)(n * f));
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < n; ++t) {
        const double* dyt = dy + t * d;
        double* dxt = dx + t * d;
        for (int64_t i = 0; i < d; ++i) dxt[i] = 0.0;
        int nent;
        if (row_nnz[t] <= k) nent = row_nnz[t];
        else if (spill_slot[t] >= 0) nent = (int)f;
        else nent = 0;
        for (int s = 0; s < nent; ++s) {
            int64_t j;
            double a, u;
            if (row_nnz[t] <= k) {
                j = ell_idx[t * k + s]; a = ell_a[t * k + s]; u = ell_u[t * k + s];
            } else {
                j = s; a = spill_a[spill_slot[t] * f + s]; u = spill_u[spill_slot[t] * f + s];
                if (!(a > 0.0)) continue;
            }
            double dh = 0.0;
            for (int64_t i = 0; i < d; ++i) dh += dyt[i] * wd[j * d + i];
            const double du = dh * a, dg = dh * u;
            du_scratch[t * f + j] = du;
            dg_scratch[t * f + j] = dg;
            for (int64_t i = 0; i < d; ++i) dxt[i] += du * wu_t[j * d + i] + dg * wg_t[j * d + i];
        }
    }
    /* weight gradients: per neuron j, sum over tokens in ascending t */
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t j = 0; j < f; ++j) {
        double* gwd = dwd + j * d;
        double* gwu = dwu_t + j * d;
        double* gwg = dwg_t + j * d;
        for (int64_t i = 0; i < d; ++i) { gwd[i] = 0.0; gwu[i] = 0.0; gwg[i] = 0.0; }
        for (int64_t t = 0; t < n; ++t) {
            const double du = du_scratch[t * f + j], dg = dg_scratch[t * f + j];
            /* look the entry up directly: it may be active with dh = 0, and
             * h dy is still needed for dW_down then */
            double a = 0.0, u = 0.0;
            if (row_nnz[t] <= k) {
                for (int s = 0; s < row_nnz[t]; ++s)
                    if (ell_idx[t * k + s] == j) { a = ell_a[t * k + s]; u = ell_u[t * k + s]; break; }
            } else if (spill_slot[t] >= 0) {
                a = spill_a[spill_slot[t] * f + j];
                u = spill_u[spill_slot[t] * f + j];
            }
            if (!(a > 0.0)) continue;
            const double h = a * u;
            const double* xt = x + t * d;
            const double* dyt = dy + t * d;
            for (int64_t i = 0; i < d; ++i) {
                gwd[i] += h * dyt[i];
                gwu[i] += du * xt[i];
                gwg[i] += dg * xt[i];
            }
        }
    }
}
