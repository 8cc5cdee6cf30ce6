/*
 * twell_oracle.c -- plain, slow, single-threaded fp64 CPU oracle for the
 * activation-sparse gated FFN and its TwELL / hybrid sparse formats.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * bench's CPU-baseline leg may load this library.  The product path (the CUDA
 * library) never links, loads or calls it, and shares no code with it.
 *
 * Source of the method: the technical summary page of "Sparser, Faster,
 * Lighter Transformer Language Models" (arXiv 2603.23198, gist.science),
 * cited below as [SFL <section>].  The page describes the method in prose
 * only; every function states which passage it follows and which reading of
 * an open point it takes.
 *
 * Conventions shared by every function (all readings of points the page
 * leaves open):
 *   - Floating point is fp64 throughout.  Inputs are the exact widening of
 *     the caller's (bf16- or fp32-rounded) tensors.
 *   - x is [T][d] row-major.  The three weights are passed as [F][d]
 *     row-major: Wg_t[j][i] is the gate weight from input i to unit j,
 *     Wu_t[j][i] the up weight, Wd[j][c] the down weight from unit j to
 *     output c.  Row j of each is unit j's d-vector.
 *   - sigma (the gate activation) is ReLU: g = z > 0 ? z : +0.0  [SFL 2.1,
 *     last bullet; 2.2 names the gate sigma(x Wg)].
 *   - "Non-zero" means the stored value compares unequal to 0.
 *   - TwELL tiles hold columns [k*W, (k+1)*W); inside a tile the non-zeros
 *     are packed in ascending column order; unused slots hold (+0, 0).
 *   - TwELL arrays are tile-major: val/idx [K][T][C], cnt/spill_ref [K][T].
 *   - cnt holds the TRUE number of non-zeros of (t,k), which may exceed C.
 *     When it does, the first C non-zeros still fill the slots and the whole
 *     W-wide dense segment of (t,k) is copied to a spill list.  The page does
 *     not say what happens on overflow; spilling keeps the format lossless.
 *   - Hybrid rows: a row with nnz <= C_h is an ELL row (global indices,
 *     ascending, padded with (+0, 0)); a row with nnz > C_h is a dense
 *     backup row.  Backup slots are numbered in ascending token order.
 *   - u ("up" activation) is saved only on the hybrid pattern: at positions
 *     where g == 0 the saved u is +0.
 *   - ReLU'(0) = 0 and sign(0) = 0; the L1 term adds lambda*sign(g) to dL/dg
 *     elementwise.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>

#define ORC_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* Storage rounding of the gate activations.  TwELL stores g in the model's  */
/* activation dtype [SFL 2.1], so in a bf16 model g is a bf16 value; the     */
/* oracle applies the same rounding to its exact fp64 g:                     */
/*   mode 0  none (exact fp64)                                               */
/*   mode 1  bf16: nearest value with 8 significant bits, ties to even       */
/*   mode 2  fp32: the C conversion to float (round to nearest even)         */
/* Inputs here are finite and far from the bf16/fp32 range limits.           */
/* ------------------------------------------------------------------------ */
ORC_API double orc_round_storage(double v, int mode)
{
    if (mode == 1) {
        if (v == 0.0) return v;
        int e;
        double m = frexp(v, &e);          /* v = m * 2^e, 0.5 <= |m| < 1 */
        double q = nearbyint(m * 256.0);  /* default mode: nearest, ties to even */
        return ldexp(q, e - 8);
    }
    if (mode == 2) return (double)(float)v;
    return v;
}

/* ------------------------------------------------------------------------ */
/* Dense FFN, the plain definition of what the sparse path computes.        */
/* [SFL 2.2]: up projection x Wu, gate activation sigma(x Wg), down         */
/* projection h Wd with h = sigma(x Wg) * (x Wu) elementwise.                */
/* g is rounded to its storage dtype (g_round, see orc_round_storage); u, h  */
/* and y stay exact.  Any output pointer may be NULL.                        */
/* ------------------------------------------------------------------------ */
ORC_API void orc_dense_ffn(int T, int d, int F,
                           const double* x, const double* Wg_t,
                           const double* Wu_t, const double* Wd, int g_round,
                           double* z_out, double* g_out, double* u_out,
                           double* y_out)
{
    for (int t = 0; t < T; ++t) {
        const double* xt = x + (size_t)t * d;
        if (y_out)
            for (int c = 0; c < d; ++c) y_out[(size_t)t * d + c] = 0.0;
        for (int j = 0; j < F; ++j) {
            const double* wg = Wg_t + (size_t)j * d;
            const double* wu = Wu_t + (size_t)j * d;
            double z = 0.0, u = 0.0;
            for (int i = 0; i < d; ++i) {
                z += xt[i] * wg[i];
                u += xt[i] * wu[i];
            }
            double g = orc_round_storage(z > 0.0 ? z : 0.0, g_round);
            if (z_out) z_out[(size_t)t * F + j] = z;
            if (g_out) g_out[(size_t)t * F + j] = g;
            if (u_out) u_out[(size_t)t * F + j] = u;
            if (y_out && g != 0.0) {
                double h = g * u;
                const double* wd = Wd + (size_t)j * d;
                for (int c = 0; c < d; ++c) y_out[(size_t)t * d + c] += h * wd[c];
            }
        }
    }
}

/* Gate only: g = relu(x Wg), rounded to storage, for a subset of rows     */
/* (rows[r] indexes x).                                                      */
ORC_API void orc_gate_rows(int R, const int32_t* rows, int d, int F,
                           const double* x, const double* Wg_t, int g_round,
                           double* g_out)
{
    for (int r = 0; r < R; ++r) {
        const double* xt = x + (size_t)rows[r] * d;
        for (int j = 0; j < F; ++j) {
            const double* wg = Wg_t + (size_t)j * d;
            double z = 0.0;
            for (int i = 0; i < d; ++i) z += xt[i] * wg[i];
            g_out[(size_t)r * F + j] = orc_round_storage(z > 0.0 ? z : 0.0, g_round);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* TwELL encode [SFL 2.1]: columns are cut into tiles of width W and each    */
/* row's non-zeros are packed, with tile-local indices, inside each tile.    */
/* Returns the number of spill entries needed (entries beyond spill_cap are  */
/* counted but not written).  Spill entries are numbered in (k, t) order.    */
/* ------------------------------------------------------------------------ */
ORC_API int32_t orc_twell_encode(int T, int F, int W, int C, const double* g,
                                 double* val, uint8_t* idx, uint8_t* cnt,
                                 int32_t* spill_ref, int32_t spill_cap,
                                 int32_t* spill_tk, double* spill_val)
{
    int K = F / W;
    int32_t n_spill = 0;
    for (int k = 0; k < K; ++k) {
        for (int t = 0; t < T; ++t) {
            size_t kt = (size_t)k * T + t;
            const double* seg = g + (size_t)t * F + (size_t)k * W;
            for (int s = 0; s < C; ++s) {
                val[kt * C + s] = 0.0;
                idx[kt * C + s] = 0;
            }
            int n = 0;
            for (int c = 0; c < W; ++c) {
                if (seg[c] != 0.0) {
                    if (n < C) {
                        val[kt * C + n] = seg[c];
                        idx[kt * C + n] = (uint8_t)c;
                    }
                    ++n;
                }
            }
            cnt[kt] = (uint8_t)n;
            if (n > C) {
                if (n_spill < spill_cap) {
                    spill_ref[kt] = n_spill;
                    spill_tk[2 * (size_t)n_spill + 0] = t;
                    spill_tk[2 * (size_t)n_spill + 1] = k;
                    for (int c = 0; c < W; ++c)
                        spill_val[(size_t)n_spill * W + c] = seg[c];
                }
                ++n_spill;
            }
        }
    }
    return n_spill;
}

/* TwELL decode: the inverse of the encoding above, into a dense [T][F]. */
ORC_API void orc_twell_decode(int T, int F, int W, int C, const double* val,
                              const uint8_t* idx, const uint8_t* cnt,
                              const int32_t* spill_ref, const double* spill_val,
                              double* g)
{
    int K = F / W;
    for (size_t e = 0; e < (size_t)T * F; ++e) g[e] = 0.0;
    for (int k = 0; k < K; ++k) {
        for (int t = 0; t < T; ++t) {
            size_t kt = (size_t)k * T + t;
            double* seg = g + (size_t)t * F + (size_t)k * W;
            int n = cnt[kt];
            if (n <= C) {
                for (int s = 0; s < n; ++s) seg[idx[kt * C + s]] = val[kt * C + s];
            } else {
                const double* sp = spill_val + (size_t)spill_ref[kt] * W;
                for (int c = 0; c < W; ++c) seg[c] = sp[c];
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Sparse FFN from TwELL [SFL 2.2]: only the active units' weights are used;  */
/* per active unit j a dot product u = x_t . Wu_t[j] and a scaled row        */
/* y_t += (g * u) Wd[j] are accumulated.                                     */
/* ------------------------------------------------------------------------ */
static void orc_unit_contrib(int d, const double* xt, double gv,
                             const double* wu, const double* wd, double* yt)
{
    double u = 0.0;
    for (int i = 0; i < d; ++i) u += xt[i] * wu[i];
    double h = gv * u;
    for (int c = 0; c < d; ++c) yt[c] += h * wd[c];
}

ORC_API void orc_twell_ffn(int T, int d, int F, int W, int C,
                           const double* x, const double* val,
                           const uint8_t* idx, const uint8_t* cnt,
                           const int32_t* spill_ref, const double* spill_val,
                           const double* Wu_t, const double* Wd, double* y)
{
    int K = F / W;
    for (int t = 0; t < T; ++t) {
        const double* xt = x + (size_t)t * d;
        double* yt = y + (size_t)t * d;
        for (int c = 0; c < d; ++c) yt[c] = 0.0;
        for (int k = 0; k < K; ++k) {
            size_t kt = (size_t)k * T + t;
            int n = cnt[kt];
            if (n <= C) {
                for (int s = 0; s < n; ++s) {
                    int j = k * W + idx[kt * C + s];
                    orc_unit_contrib(d, xt, val[kt * C + s], Wu_t + (size_t)j * d,
                                     Wd + (size_t)j * d, yt);
                }
            } else {
                const double* sp = spill_val + (size_t)spill_ref[kt] * W;
                for (int c = 0; c < W; ++c) {
                    if (sp[c] == 0.0) continue;
                    int j = k * W + c;
                    orc_unit_contrib(d, xt, sp[c], Wu_t + (size_t)j * d,
                                     Wd + (size_t)j * d, yt);
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Hybrid split [SFL 2.3]: rows with few non-zeros go to a compact ELL part, */
/* rows with too many go to dense backup rows.  Works from a dense g (the    */
/* decoded TwELL).  Returns the number of backup rows needed.                */
/* ------------------------------------------------------------------------ */
ORC_API int32_t orc_hybrid_split(int T, int F, int C_h, const double* g,
                                 double* ell_g, uint16_t* ell_idx,
                                 int32_t* row_nnz, int32_t* row_slot,
                                 int32_t backup_cap, int32_t* backup_rows,
                                 double* backup_g)
{
    int32_t n_backup = 0;
    for (int t = 0; t < T; ++t) {
        const double* gt = g + (size_t)t * F;
        int n = 0;
        for (int j = 0; j < F; ++j) n += (gt[j] != 0.0);
        row_nnz[t] = n;
        for (int s = 0; s < C_h; ++s) {
            ell_g[(size_t)t * C_h + s] = 0.0;
            ell_idx[(size_t)t * C_h + s] = 0;
        }
        if (n <= C_h) {
            row_slot[t] = -1;
            int s = 0;
            for (int j = 0; j < F; ++j) {
                if (gt[j] != 0.0) {
                    ell_g[(size_t)t * C_h + s] = gt[j];
                    ell_idx[(size_t)t * C_h + s] = (uint16_t)j;
                    ++s;
                }
            }
        } else {
            row_slot[t] = n_backup;
            if (n_backup < backup_cap) {
                backup_rows[n_backup] = t;
                for (int j = 0; j < F; ++j) backup_g[(size_t)n_backup * F + j] = gt[j];
            }
            ++n_backup;
        }
    }
    return n_backup;
}

/* Dense g from a hybrid (inverse of the split). */
ORC_API void orc_hybrid_decode(int T, int F, int C_h, const double* ell_g,
                               const uint16_t* ell_idx, const int32_t* row_slot,
                               const double* backup_g, double* g)
{
    for (int t = 0; t < T; ++t) {
        double* gt = g + (size_t)t * F;
        for (int j = 0; j < F; ++j) gt[j] = 0.0;
        if (row_slot[t] < 0) {
            for (int s = 0; s < C_h; ++s) {
                double v = ell_g[(size_t)t * C_h + s];
                if (v != 0.0) gt[ell_idx[(size_t)t * C_h + s]] = v;
            }
        } else {
            const double* b = backup_g + (size_t)row_slot[t] * F;
            for (int j = 0; j < F; ++j) gt[j] = b[j];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Training forward on the hybrid pattern [SFL 2.3, 2.4]: u = x Wu sampled   */
/* at the active positions (ELL slots, or non-zero entries of a backup row),  */
/* then y = (g * u) Wd.  ell_u / backup_u receive u on the pattern (+0 off   */
/* the pattern).  n_backup = number of valid backup rows.                    */
/* ------------------------------------------------------------------------ */
ORC_API void orc_hybrid_forward(int T, int d, int F, int C_h,
                                const double* x, const double* ell_g,
                                const uint16_t* ell_idx, const int32_t* row_slot,
                                const double* backup_g, const double* Wu_t,
                                const double* Wd, double* ell_u,
                                double* backup_u, double* y)
{
    for (int t = 0; t < T; ++t) {
        const double* xt = x + (size_t)t * d;
        double* yt = y + (size_t)t * d;
        for (int c = 0; c < d; ++c) yt[c] = 0.0;
        int slot = row_slot[t];
        int n_items = slot < 0 ? C_h : F;
        if (slot >= 0) /* the ELL slots of a backup row are off the pattern */
            for (int s = 0; s < C_h; ++s) ell_u[(size_t)t * C_h + s] = 0.0;
        for (int s = 0; s < n_items; ++s) {
            double gv;
            int j;
            if (slot < 0) {
                gv = ell_g[(size_t)t * C_h + s];
                j = ell_idx[(size_t)t * C_h + s];
            } else {
                gv = backup_g[(size_t)slot * F + s];
                j = s;
            }
            double u = 0.0;
            if (gv != 0.0) {
                const double* wu = Wu_t + (size_t)j * d;
                for (int i = 0; i < d; ++i) u += xt[i] * wu[i];
                double h = gv * u;
                const double* wd = Wd + (size_t)j * d;
                for (int c = 0; c < d; ++c) yt[c] += h * wd[c];
            }
            if (slot < 0) ell_u[(size_t)t * C_h + s] = u;
            else backup_u[(size_t)slot * F + s] = u;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Backward of the gated FFN with the L1 activation term [SFL 2.4, 3].       */
/* Loss L = sum(y * dy) + lambda * sum(g) (g >= 0, so sum(g) = ||g||_1).      */
/* For every active (t, j) with saved g > 0 and u:                          */
/*   dh = dy_t . Wd[j]            du = dh * g                                 */
/*   dz = dh * u + lambda         (the ReLU mask is 1 because g > 0)          */
/*   dx_t    += du * Wu_t[j] + dz * Wg_t[j]                                   */
/*   dWd[j]  += (g * u) * dy_t                                                */
/*   dWu_t[j] += du * x_t         dWg_t[j] += dz * x_t                        */
/* Inactive entries contribute nothing (ReLU'(0) = 0, sign(0) = 0).          */
/* ------------------------------------------------------------------------ */
static void orc_backward_entry(int d, const double* xt, const double* dyt,
                               double gv, double uv, double lambda,
                               const double* wg, const double* wu, const double* wd,
                               double* dxt, double* dwg, double* dwu, double* dwd)
{
    double dh = 0.0;
    for (int c = 0; c < d; ++c) dh += dyt[c] * wd[c];
    double du = dh * gv;
    double dz = dh * uv + lambda;
    double h = gv * uv;
    for (int i = 0; i < d; ++i) {
        dxt[i] += du * wu[i] + dz * wg[i];
        dwu[i] += du * xt[i];
        dwg[i] += dz * xt[i];
        dwd[i] += h * dyt[i];
    }
}

ORC_API void orc_hybrid_backward(int T, int d, int F, int C_h,
                                 const double* x, const double* dy,
                                 const double* ell_g, const double* ell_u,
                                 const uint16_t* ell_idx, const int32_t* row_slot,
                                 const double* backup_g, const double* backup_u,
                                 const double* Wg_t, const double* Wu_t,
                                 const double* Wd, double lambda,
                                 double* dx, double* dWg_t, double* dWu_t,
                                 double* dWd)
{
    memset(dx, 0, sizeof(double) * (size_t)T * d);
    memset(dWg_t, 0, sizeof(double) * (size_t)F * d);
    memset(dWu_t, 0, sizeof(double) * (size_t)F * d);
    memset(dWd, 0, sizeof(double) * (size_t)F * d);
    for (int t = 0; t < T; ++t) {
        int slot = row_slot[t];
        int n_items = slot < 0 ? C_h : F;
        for (int s = 0; s < n_items; ++s) {
            double gv, uv;
            int j;
            if (slot < 0) {
                gv = ell_g[(size_t)t * C_h + s];
                uv = ell_u[(size_t)t * C_h + s];
                j = ell_idx[(size_t)t * C_h + s];
            } else {
                gv = backup_g[(size_t)slot * F + s];
                uv = backup_u[(size_t)slot * F + s];
                j = s;
            }
            if (!(gv > 0.0)) continue;
            orc_backward_entry(d, x + (size_t)t * d, dy + (size_t)t * d, gv, uv,
                               lambda, Wg_t + (size_t)j * d, Wu_t + (size_t)j * d,
                               Wd + (size_t)j * d, dx + (size_t)t * d,
                               dWg_t + (size_t)j * d, dWu_t + (size_t)j * d,
                               dWd + (size_t)j * d);
        }
    }
}

/* Dense backward: the same loss, computed from x and the weights alone by   */
/* the textbook chain rule over every (t, j), with no sparse format.          */
ORC_API void orc_dense_ffn_backward(int T, int d, int F, const double* x,
                                    const double* Wg_t, const double* Wu_t,
                                    const double* Wd, const double* dy,
                                    double lambda, double* dx, double* dWg_t,
                                    double* dWu_t, double* dWd)
{
    memset(dx, 0, sizeof(double) * (size_t)T * d);
    memset(dWg_t, 0, sizeof(double) * (size_t)F * d);
    memset(dWu_t, 0, sizeof(double) * (size_t)F * d);
    memset(dWd, 0, sizeof(double) * (size_t)F * d);
    for (int t = 0; t < T; ++t) {
        const double* xt = x + (size_t)t * d;
        const double* dyt = dy + (size_t)t * d;
        for (int j = 0; j < F; ++j) {
            const double* wg = Wg_t + (size_t)j * d;
            const double* wu = Wu_t + (size_t)j * d;
            const double* wd = Wd + (size_t)j * d;
            double z = 0.0, u = 0.0, dh = 0.0;
            for (int i = 0; i < d; ++i) {
                z += xt[i] * wg[i];
                u += xt[i] * wu[i];
                dh += dyt[i] * wd[i];
            }
            double g = z > 0.0 ? z : 0.0;
            double relu_grad = z > 0.0 ? 1.0 : 0.0;
            double sign_g = g > 0.0 ? 1.0 : 0.0;
            double h = g * u;
            double du = dh * g;                       /* dL/du */
            double dg = dh * u + lambda * sign_g;     /* dL/dg */
            double dz = dg * relu_grad;               /* dL/dz */
            for (int i = 0; i < d; ++i) {
                dx[(size_t)t * d + i] += du * wu[i] + dz * wg[i];
                dWu_t[(size_t)j * d + i] += du * xt[i];
                dWg_t[(size_t)j * d + i] += dz * xt[i];
                dWd[(size_t)j * d + i] += h * dyt[i];
            }
        }
    }
}
