/*
 * Oracle for multi-scale deformable attention and BEVFormer Spatial
 * Cross-Attention: plain CPU loops in double precision, written from the
 * equations of the pages (see msda_oracle.h for the sources and the
 * conventions).  TEST INFRASTRUCTURE ONLY: nothing on the product path may
 * call it.  Deliberately unoptimised: one loop per index of the equations,
 * no blocking, no fusion, no reordering.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off (no -ffast-math),
 * so that the binary32 steps of the corner decision are single IEEE
 * operations with round-to-nearest.
 */
#include "msda_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Argument checks                                                          */
/* ------------------------------------------------------------------------ */

static int check_levels(int Nv, int L, const int64_t* shapes, const int64_t* starts)
{
    if (L < 1 || shapes == NULL || starts == NULL) return -1;
    for (int l = 0; l < L; ++l) {
        int64_t Hl = shapes[2 * l], Wl = shapes[2 * l + 1];
        if (Hl < 1 || Wl < 1) return -1;
        if (starts[l] < 0 || starts[l] + Hl * Wl > (int64_t)Nv) return -1;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Softmax ([BQ] 4.2): each head normalises its own L*P logits;             */
/* the weights of one group sum to one.                                     */
/* ------------------------------------------------------------------------ */

int oracle_softmax(const double* logits, int64_t groups, int n, double* alpha)
{
    if (logits == NULL || alpha == NULL || groups < 0 || n < 1) return -1;
    for (int64_t g = 0; g < groups; ++g) {
        const double* a = logits + g * n;
        double* w = alpha + g * n;
        double m = a[0];
        for (int i = 1; i < n; ++i)
            if (a[i] > m) m = a[i];
        double z = 0.0;
        for (int i = 0; i < n; ++i) {
            w[i] = exp(a[i] - m);
            z += w[i];
        }
        for (int i = 0; i < n; ++i) w[i] /= z;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Location ([BQ] 5): s = rho_{m(k)} + (dx / W_l, dy / H_l), m(k) = k mod R.  */
/* ------------------------------------------------------------------------ */

static double fused_location(double rho, double d, int64_t n, int coord_f32)
{
    if (coord_f32) {
        volatile float q = (float)d / (float)n;
        volatile float s = (float)rho + q;
        return (double)s;
    }
    return rho + d / (double)n;
}

/* Continuous pixel coordinate on an axis of n pixels ([BQ] 6): n*s - 1/2. */
static double pixel_coord(double s, int64_t n, int coord_f32)
{
    if (coord_f32) {
        volatile float prod = (float)n * (float)s;
        volatile float c = prod - 0.5f;
        return (double)c;
    }
    return (double)n * s - 0.5;
}

/* ------------------------------------------------------------------------ */
/* Bilinear neighbourhood ([BQ] 6, four-neighbour interpolation).           */
/* Neighbour g = 0..3 is (x0 + (g & 1), y0 + (g >> 1)), x0 = floor(x),       */
/* y0 = floor(y), with weight ((g&1) ? lx : 1-lx) * ((g>>1) ? ly : 1-ly).    */
/* A neighbour outside the map reads zero (zero padding).                   */
/* ------------------------------------------------------------------------ */

typedef struct {
    int valid;       /* 0: no neighbour of non-zero weight lies in the map */
    double lx, ly;   /* fractional parts x - x0, y - y0 */
    int64_t row[4];  /* value row of each neighbour, -1 when outside */
} corners_t;

static corners_t locate(double x, double y, int64_t Hl, int64_t Wl, int64_t start)
{
    corners_t c;
    c.valid = 0;
    c.lx = c.ly = 0.0;
    for (int g = 0; g < 4; ++g) c.row[g] = -1;
    /* For x <= -1 or x >= W every neighbour of non-zero weight is outside
     * the map, so the sample is zero either way.  The test is false for NaN,
     * so a non-finite location also reads nothing. */
    if (!(x > -1.0 && x < (double)Wl && y > -1.0 && y < (double)Hl)) return c;
    double fx = floor(x), fy = floor(y);
    int64_t x0 = (int64_t)fx, y0 = (int64_t)fy;
    c.valid = 1;
    c.lx = x - fx;
    c.ly = y - fy;
    for (int g = 0; g < 4; ++g) {
        int64_t xc = x0 + (g & 1), yc = y0 + (g >> 1);
        if (xc >= 0 && xc < Wl && yc >= 0 && yc < Hl) c.row[g] = start + yc * Wl + xc;
    }
    return c;
}

static double corner_weight(const corners_t* c, int g)
{
    double wx = (g & 1) ? c->lx : 1.0 - c->lx;
    double wy = (g >> 1) ? c->ly : 1.0 - c->ly;
    return wx * wy;
}

/* ------------------------------------------------------------------------ */
/* One query row, all heads ([BQ] 7-9):                                     */
/*   g^(h) = sum_l sum_k alpha_{h,l,k} * B(V_l^(h), s_{h,l,k}),              */
/*   out = concat_h g^(h).                                                  */
/* vb: [Nv, H, Dh] of one batch item (and camera); loc_row [H, L, P, 2];     */
/* attn_row [H, L, P]; out_row [H*Dh].                                      */
/* ------------------------------------------------------------------------ */

static void row_forward(const double* vb, int H, int Dh, int L, const int64_t* shapes,
                        const int64_t* starts, int P, const double* loc_row,
                        const double* attn_row, int coord_f32, double* out_row)
{
    for (int h = 0; h < H; ++h) {
        double* g = out_row + (int64_t)h * Dh;
        for (int d = 0; d < Dh; ++d) g[d] = 0.0;
        for (int l = 0; l < L; ++l) {
            int64_t Hl = shapes[2 * l], Wl = shapes[2 * l + 1];
            for (int k = 0; k < P; ++k) {
                int64_t s = ((int64_t)h * L + l) * P + k;
                double alpha = attn_row[s];
                double x = pixel_coord(loc_row[2 * s + 0], Wl, coord_f32);
                double y = pixel_coord(loc_row[2 * s + 1], Hl, coord_f32);
                corners_t c = locate(x, y, Hl, Wl, starts[l]);
                if (!c.valid) continue;
                for (int q = 0; q < 4; ++q) {
                    if (c.row[q] < 0) continue;
                    double w = corner_weight(&c, q);
                    const double* v = vb + (c.row[q] * H + h) * Dh;
                    for (int d = 0; d < Dh; ++d) g[d] += alpha * w * v[d];
                }
            }
        }
    }
}

/* Derivative of row_forward for one row, given the upstream gradient of
 * out_row.  Accumulates into gvb [Nv, H, Dh]; overwrites gloc_row [H, L, P, 2]
 * and gattn_row [H, L, P].
 *   f = sum_g w_g V_g                       (the bilinear read)
 *   d out / d alpha = f
 *   d f / d x = (1-ly)(V_10 - V_00) + ly (V_11 - V_01)
 *   d f / d y = (1-lx)(V_01 - V_00) + lx (V_11 - V_10)
 *   d x / d s_x = W_l,  d y / d s_y = H_l   (x = W_l s_x - 1/2)
 * with V_g = 0 for a neighbour outside the map.  At an integer coordinate the
 * derivative is the one of the cell that floor() selects. */
static void row_backward(const double* vb, int H, int Dh, int L, const int64_t* shapes,
                         const int64_t* starts, int P, const double* loc_row,
                         const double* attn_row, const double* gout_row, int coord_f32,
                         double* gvb, double* gloc_row, double* gattn_row)
{
    for (int h = 0; h < H; ++h) {
        const double* go = gout_row + (int64_t)h * Dh;
        for (int l = 0; l < L; ++l) {
            int64_t Hl = shapes[2 * l], Wl = shapes[2 * l + 1];
            for (int k = 0; k < P; ++k) {
                int64_t s = ((int64_t)h * L + l) * P + k;
                double alpha = attn_row[s];
                double x = pixel_coord(loc_row[2 * s + 0], Wl, coord_f32);
                double y = pixel_coord(loc_row[2 * s + 1], Hl, coord_f32);
                corners_t c = locate(x, y, Hl, Wl, starts[l]);
                gattn_row[s] = 0.0;
                gloc_row[2 * s + 0] = 0.0;
                gloc_row[2 * s + 1] = 0.0;
                if (!c.valid) continue;
                /* dot[g] = <grad_out, V_g>, zero for an outside neighbour */
                double dot[4] = {0.0, 0.0, 0.0, 0.0};
                for (int q = 0; q < 4; ++q) {
                    if (c.row[q] < 0) continue;
                    const double* v = vb + (c.row[q] * H + h) * Dh;
                    for (int d = 0; d < Dh; ++d) dot[q] += go[d] * v[d];
                }
                double gw = 0.0;
                for (int q = 0; q < 4; ++q) gw += corner_weight(&c, q) * dot[q];
                gattn_row[s] = gw;
                double dfdx = (1.0 - c.ly) * (dot[1] - dot[0]) + c.ly * (dot[3] - dot[2]);
                double dfdy = (1.0 - c.lx) * (dot[2] - dot[0]) + c.lx * (dot[3] - dot[1]);
                gloc_row[2 * s + 0] = alpha * (double)Wl * dfdx;
                gloc_row[2 * s + 1] = alpha * (double)Hl * dfdy;
                for (int q = 0; q < 4; ++q) {
                    if (c.row[q] < 0) continue;
                    double w = alpha * corner_weight(&c, q);
                    double* gv = gvb + (c.row[q] * H + h) * Dh;
                    for (int d = 0; d < Dh; ++d) gv[d] += w * go[d];
                }
            }
        }
    }
}

/* Locations and weights of one query row from its reference points, pixel
 * offsets and logits ([BQ] 4.2, 5, 18.4).  ref_row [R, 2]; off_row
 * [H, L, P, 2]; logit_row [H, L, P] -> loc_row [H, L, P, 2], attn_row [H, L, P]. */
static void row_locations(int H, int L, const int64_t* shapes, int P, int R,
                          const double* ref_row, const double* off_row,
                          const double* logit_row, int coord_f32,
                          double* loc_row, double* attn_row)
{
    oracle_softmax(logit_row, H, L * P, attn_row);
    for (int h = 0; h < H; ++h)
        for (int l = 0; l < L; ++l) {
            int64_t Hl = shapes[2 * l], Wl = shapes[2 * l + 1];
            for (int k = 0; k < P; ++k) {
                int64_t s = ((int64_t)h * L + l) * P + k;
                int m = k % R;
                loc_row[2 * s + 0] = fused_location(ref_row[2 * m + 0], off_row[2 * s + 0], Wl, coord_f32);
                loc_row[2 * s + 1] = fused_location(ref_row[2 * m + 1], off_row[2 * s + 1], Hl, coord_f32);
            }
        }
}

/* ------------------------------------------------------------------------ */
/* MSDA entry points                                                        */
/* ------------------------------------------------------------------------ */

static int check_msda(const double* value, int B, int Nv, int H, int Dh, int L,
                      const int64_t* shapes, const int64_t* starts, int Nq, int P)
{
    if (value == NULL || B < 0 || Nv < 1 || H < 1 || Dh < 1 || Nq < 0 || P < 1) return -1;
    return check_levels(Nv, L, shapes, starts);
}

int oracle_msda_forward(const double* value, int B, int Nv, int H, int Dh,
                        int L, const int64_t* shapes, const int64_t* starts,
                        int Nq, int P, const double* loc, const double* attn,
                        int coord_f32, double* out)
{
    if (check_msda(value, B, Nv, H, Dh, L, shapes, starts, Nq, P)) return -1;
    if (loc == NULL || attn == NULL || out == NULL) return -1;
    const int64_t S = (int64_t)H * L * P;
    for (int b = 0; b < B; ++b)
        for (int q = 0; q < Nq; ++q) {
            int64_t r = (int64_t)b * Nq + q;
            row_forward(value + (int64_t)b * Nv * H * Dh, H, Dh, L, shapes, starts, P,
                        loc + r * S * 2, attn + r * S, coord_f32, out + r * H * Dh);
        }
    return 0;
}

int oracle_fused_locations(int B, int H, int L, const int64_t* shapes,
                           int Nq, int P, int R, const double* ref,
                           const double* off, const double* logits,
                           int coord_f32, double* loc, double* attn)
{
    if (B < 0 || H < 1 || L < 1 || shapes == NULL || Nq < 0 || P < 1 || R < 1 || P % R)
        return -1;
    if (ref == NULL || off == NULL || logits == NULL || loc == NULL || attn == NULL) return -1;
    const int64_t S = (int64_t)H * L * P;
    for (int b = 0; b < B; ++b)
        for (int q = 0; q < Nq; ++q) {
            int64_t r = (int64_t)b * Nq + q;
            row_locations(H, L, shapes, P, R, ref + r * R * 2, off + r * S * 2,
                          logits + r * S, coord_f32, loc + r * S * 2, attn + r * S);
        }
    return 0;
}

int oracle_msda_forward_fused(const double* value, int B, int Nv, int H, int Dh,
                              int L, const int64_t* shapes, const int64_t* starts,
                              int Nq, int P, int R, const double* ref,
                              const double* off, const double* logits,
                              int coord_f32, double* out)
{
    if (check_msda(value, B, Nv, H, Dh, L, shapes, starts, Nq, P)) return -1;
    if (out == NULL) return -1;
    const int64_t S = (int64_t)H * L * P;
    double* loc = (double*)malloc(sizeof(double) * (size_t)(B * (int64_t)Nq * S * 2 + 1));
    double* attn = (double*)malloc(sizeof(double) * (size_t)(B * (int64_t)Nq * S + 1));
    int rc = -1;
    if (loc && attn &&
        oracle_fused_locations(B, H, L, shapes, Nq, P, R, ref, off, logits, coord_f32, loc, attn) == 0)
        rc = oracle_msda_forward(value, B, Nv, H, Dh, L, shapes, starts, Nq, P, loc, attn,
                                 coord_f32, out);
    free(loc);
    free(attn);
    return rc;
}

int oracle_msda_backward(const double* value, int B, int Nv, int H, int Dh,
                         int L, const int64_t* shapes, const int64_t* starts,
                         int Nq, int P, const double* loc, const double* attn,
                         const double* grad_out, int coord_f32,
                         double* grad_value, double* grad_loc, double* grad_attn)
{
    if (check_msda(value, B, Nv, H, Dh, L, shapes, starts, Nq, P)) return -1;
    if (!loc || !attn || !grad_out || !grad_value || !grad_loc || !grad_attn) return -1;
    const int64_t S = (int64_t)H * L * P;
    const int64_t VB = (int64_t)Nv * H * Dh;
    memset(grad_value, 0, sizeof(double) * (size_t)(B * VB));
    for (int b = 0; b < B; ++b)
        for (int q = 0; q < Nq; ++q) {
            int64_t r = (int64_t)b * Nq + q;
            row_backward(value + b * VB, H, Dh, L, shapes, starts, P, loc + r * S * 2,
                         attn + r * S, grad_out + r * H * Dh, coord_f32, grad_value + b * VB,
                         grad_loc + r * S * 2, grad_attn + r * S);
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* SCA ([SCA] rebatch and average listings; [BQ] 10)                        */
/* ------------------------------------------------------------------------ */

/* A camera hits query q when any of the R anchors of q is valid in it (the
 * rebatch listing sums the mask over its last axis and keeps the non-zero
 * entries).  The hit queries of one (batch, camera) are listed in ascending
 * order, as nonzero() returns them. */
int oracle_sca_compact(const uint8_t* bev_mask, int Ncam, int B, int Nq, int R,
                       int32_t* idx, int32_t* count, int32_t* pos, int32_t* hits)
{
    if (!bev_mask || !idx || !count || !pos || !hits || Ncam < 1 || B < 0 || Nq < 0 || R < 1)
        return -1;
    for (int b = 0; b < B; ++b)
        for (int q = 0; q < Nq; ++q) hits[(int64_t)b * Nq + q] = 0;
    for (int b = 0; b < B; ++b)
        for (int c = 0; c < Ncam; ++c) {
            int64_t bc = (int64_t)b * Ncam + c;
            int32_t n = 0;
            for (int q = 0; q < Nq; ++q) {
                int hit = 0;
                for (int r = 0; r < R; ++r)
                    if (bev_mask[(((int64_t)c * B + b) * Nq + q) * R + r] != 0) hit = 1;
                if (hit) {
                    idx[bc * Nq + n] = q;
                    pos[bc * Nq + q] = n;
                    n += 1;
                    hits[(int64_t)b * Nq + q] += 1;
                } else {
                    pos[bc * Nq + q] = -1;
                }
            }
            count[bc] = n;
            for (int i = n; i < Nq; ++i) idx[bc * Nq + i] = -1;
        }
    return 0;
}

typedef struct {
    int32_t *idx, *count, *pos, *hits;
    double *loc_row, *attn_row, *row;
} sca_scratch_t;

static void scratch_free(sca_scratch_t* s)
{
    free(s->idx); free(s->count); free(s->pos); free(s->hits);
    free(s->loc_row); free(s->attn_row); free(s->row);
}

static int scratch_alloc(sca_scratch_t* s, int B, int Ncam, int Nq, int64_t S, int64_t HD)
{
    s->idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)((int64_t)B * Ncam * Nq + 1));
    s->count = (int32_t*)malloc(sizeof(int32_t) * (size_t)((int64_t)B * Ncam + 1));
    s->pos = (int32_t*)malloc(sizeof(int32_t) * (size_t)((int64_t)B * Ncam * Nq + 1));
    s->hits = (int32_t*)malloc(sizeof(int32_t) * (size_t)((int64_t)B * Nq + 1));
    s->loc_row = (double*)malloc(sizeof(double) * (size_t)(S * 2));
    s->attn_row = (double*)malloc(sizeof(double) * (size_t)S);
    s->row = (double*)malloc(sizeof(double) * (size_t)HD);
    if (!s->idx || !s->count || !s->pos || !s->hits || !s->loc_row || !s->attn_row || !s->row) {
        scratch_free(s);
        return -1;
    }
    return 0;
}

static int check_sca(const double* value, int B, int Ncam, int Nv, int H, int Dh, int L,
                     const int64_t* shapes, const int64_t* starts, int Nq, int P, int R,
                     const double* ref_cam, const uint8_t* bev_mask, const double* off,
                     const double* logits)
{
    if (check_msda(value, B, Nv, H, Dh, L, shapes, starts, Nq, P)) return -1;
    if (Ncam < 1 || R < 1 || P % R || !ref_cam || !bev_mask || !off || !logits) return -1;
    return 0;
}

int oracle_sca_forward(const double* value, int B, int Ncam, int Nv, int H, int Dh,
                       int L, const int64_t* shapes, const int64_t* starts,
                       int Nq, int P, int R, const double* ref_cam,
                       const uint8_t* bev_mask, const double* off,
                       const double* logits, int coord_f32,
                       double* out, double* out_rb)
{
    if (check_sca(value, B, Ncam, Nv, H, Dh, L, shapes, starts, Nq, P, R, ref_cam, bev_mask,
                  off, logits) || out == NULL)
        return -1;
    const int64_t S = (int64_t)H * L * P, HD = (int64_t)H * Dh, VB = (int64_t)Nv * HD;
    sca_scratch_t sc;
    if (scratch_alloc(&sc, B, Ncam, Nq, S, HD)) return -1;
    oracle_sca_compact(bev_mask, Ncam, B, Nq, R, sc.idx, sc.count, sc.pos, sc.hits);

    for (int64_t i = 0; i < (int64_t)B * Nq * HD; ++i) out[i] = 0.0;
    if (out_rb)
        for (int64_t i = 0; i < (int64_t)B * Ncam * Nq * HD; ++i) out_rb[i] = 0.0;

    for (int b = 0; b < B; ++b)
        for (int c = 0; c < Ncam; ++c) {          /* ascending camera order */
            int64_t bc = (int64_t)b * Ncam + c;
            const double* vbc = value + bc * VB;
            for (int i = 0; i < sc.count[bc]; ++i) {
                int q = sc.idx[bc * Nq + i];
                int64_t bq = (int64_t)b * Nq + q;
                /* offsets and logits belong to the BEV query and are the same in
                 * every camera; the reference points are the camera's own */
                const double* ref_row = ref_cam + (((int64_t)c * B + b) * Nq + q) * R * 2;
                row_locations(H, L, shapes, P, R, ref_row, off + bq * S * 2, logits + bq * S,
                              coord_f32, sc.loc_row, sc.attn_row);
                row_forward(vbc, H, Dh, L, shapes, starts, P, sc.loc_row, sc.attn_row,
                            coord_f32, sc.row);
                if (out_rb)
                    for (int64_t d = 0; d < HD; ++d) out_rb[(bc * Nq + i) * HD + d] = sc.row[d];
                for (int64_t d = 0; d < HD; ++d) out[bq * HD + d] += sc.row[d];
            }
        }
    /* average over the cameras that hit the query, at least one */
    for (int b = 0; b < B; ++b)
        for (int q = 0; q < Nq; ++q) {
            int64_t bq = (int64_t)b * Nq + q;
            int n = sc.hits[bq] > 1 ? sc.hits[bq] : 1;
            for (int64_t d = 0; d < HD; ++d) out[bq * HD + d] /= (double)n;
        }
    scratch_free(&sc);
    return 0;
}

int oracle_sca_camera_average(const double* out_rb, const int32_t* pos, const int32_t* hits,
                              int B, int Ncam, int Nq, int64_t HD, double* out)
{
    if (out_rb == NULL || pos == NULL || hits == NULL || out == NULL || B < 0 || Ncam < 1 ||
        Nq < 0 || HD < 1)
        return -1;
    for (int b = 0; b < B; ++b)
        for (int q = 0; q < Nq; ++q) {
            const int64_t bq = (int64_t)b * Nq + q;
            double* o = out + bq * HD;
            for (int64_t d = 0; d < HD; ++d) o[d] = 0.0;
            for (int c = 0; c < Ncam; ++c) {          /* scatter-add, ascending camera */
                const int64_t bc = (int64_t)b * Ncam + c;
                const int32_t i = pos[bc * Nq + q];
                if (i < 0) continue;
                if (i >= Nq) return -1;
                for (int64_t d = 0; d < HD; ++d) o[d] += out_rb[(bc * Nq + i) * HD + d];
            }
            const int n = hits[bq] > 1 ? hits[bq] : 1;   /* clamp(count, 1) */
            for (int64_t d = 0; d < HD; ++d) o[d] /= (double)n;
        }
    return 0;
}

int oracle_sca_backward(const double* value, int B, int Ncam, int Nv, int H, int Dh,
                        int L, const int64_t* shapes, const int64_t* starts,
                        int Nq, int P, int R, const double* ref_cam,
                        const uint8_t* bev_mask, const double* off,
                        const double* logits, const double* grad_out, int coord_f32,
                        double* grad_value, double* grad_loc_rb, double* grad_attn_rb)
{
    if (check_sca(value, B, Ncam, Nv, H, Dh, L, shapes, starts, Nq, P, R, ref_cam, bev_mask,
                  off, logits))
        return -1;
    if (!grad_out || !grad_value || !grad_loc_rb || !grad_attn_rb) return -1;
    const int64_t S = (int64_t)H * L * P, HD = (int64_t)H * Dh, VB = (int64_t)Nv * HD;
    sca_scratch_t sc;
    if (scratch_alloc(&sc, B, Ncam, Nq, S, HD)) return -1;
    oracle_sca_compact(bev_mask, Ncam, B, Nq, R, sc.idx, sc.count, sc.pos, sc.hits);

    memset(grad_value, 0, sizeof(double) * (size_t)((int64_t)B * Ncam * VB));
    memset(grad_loc_rb, 0, sizeof(double) * (size_t)((int64_t)B * Ncam * Nq * S * 2));
    memset(grad_attn_rb, 0, sizeof(double) * (size_t)((int64_t)B * Ncam * Nq * S));

    for (int b = 0; b < B; ++b)
        for (int c = 0; c < Ncam; ++c) {
            int64_t bc = (int64_t)b * Ncam + c;
            for (int i = 0; i < sc.count[bc]; ++i) {
                int q = sc.idx[bc * Nq + i];
                int64_t bq = (int64_t)b * Nq + q;
                /* the average divides every camera's row by max(1, hits) */
                int n = sc.hits[bq] > 1 ? sc.hits[bq] : 1;
                for (int64_t d = 0; d < HD; ++d) sc.row[d] = grad_out[bq * HD + d] / (double)n;
                const double* ref_row = ref_cam + (((int64_t)c * B + b) * Nq + q) * R * 2;
                row_locations(H, L, shapes, P, R, ref_row, off + bq * S * 2, logits + bq * S,
                              coord_f32, sc.loc_row, sc.attn_row);
                row_backward(value + bc * VB, H, Dh, L, shapes, starts, P, sc.loc_row,
                             sc.attn_row, sc.row, coord_f32, grad_value + bc * VB,
                             grad_loc_rb + (bc * Nq + i) * S * 2, grad_attn_rb + (bc * Nq + i) * S);
            }
        }
    scratch_free(&sc);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Dense projection ([BQ] 3, 4.1, 4.2, 11, 13)                              */
/* ------------------------------------------------------------------------ */

int oracle_linear(const double* x, const double* w, const double* bias, const double* residual,
                  int M, int N, int K, double* y)
{
    if (!x || !w || !y || M < 0 || N < 1 || K < 1) return -1;
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k) acc += x[(int64_t)m * K + k] * w[(int64_t)n * K + k];
            if (bias) acc += bias[n];
            if (residual) acc += residual[(int64_t)m * N + n];
            y[(int64_t)m * N + n] = acc;
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Gradients of the SCA inputs ([BQ] 4.2, 5, 10)                            */
/* ------------------------------------------------------------------------ */

int oracle_sca_backward_inputs(int B, int Ncam, int Nq, int H, int L, const int64_t* shapes,
                               int P, int R, const uint8_t* bev_mask, const double* logits,
                               const double* grad_loc_rb, const double* grad_attn_rb,
                               double* grad_off, double* grad_logits, double* grad_ref_cam)
{
    if (B < 0 || Ncam < 1 || Nq < 0 || H < 1 || L < 1 || P < 1 || R < 1 || P % R || !shapes ||
        !bev_mask || !logits || !grad_loc_rb || !grad_attn_rb || !grad_off || !grad_logits ||
        !grad_ref_cam)
        return -1;
    const int64_t S = (int64_t)H * L * P;
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)((int64_t)B * Ncam * Nq + 1));
    int32_t* count = (int32_t*)malloc(sizeof(int32_t) * (size_t)((int64_t)B * Ncam + 1));
    int32_t* pos = (int32_t*)malloc(sizeof(int32_t) * (size_t)((int64_t)B * Ncam * Nq + 1));
    int32_t* hits = (int32_t*)malloc(sizeof(int32_t) * (size_t)((int64_t)B * Nq + 1));
    double* G = (double*)malloc(sizeof(double) * (size_t)((int64_t)B * Nq * S + 1));
    double* alpha = (double*)malloc(sizeof(double) * (size_t)(S + 1));
    if (!idx || !count || !pos || !hits || !G || !alpha) {
        free(idx); free(count); free(pos); free(hits); free(G); free(alpha);
        return -1;
    }
    oracle_sca_compact(bev_mask, Ncam, B, Nq, R, idx, count, pos, hits);
    memset(grad_off, 0, sizeof(double) * (size_t)((int64_t)B * Nq * S * 2));
    memset(grad_ref_cam, 0, sizeof(double) * (size_t)((int64_t)Ncam * B * Nq * R * 2));
    memset(G, 0, sizeof(double) * (size_t)((int64_t)B * Nq * S));
    for (int b = 0; b < B; ++b)
        for (int c = 0; c < Ncam; ++c) {
            const int64_t bc = (int64_t)b * Ncam + c;
            for (int i = 0; i < count[bc]; ++i) {
                const int q = idx[bc * Nq + i];
                const int64_t bq = (int64_t)b * Nq + q;
                const double* gl = grad_loc_rb + (bc * Nq + i) * S * 2;
                const double* ga = grad_attn_rb + (bc * Nq + i) * S;
                double* gr = grad_ref_cam + (((int64_t)c * B + b) * Nq + q) * R * 2;
                for (int h = 0; h < H; ++h)
                    for (int l = 0; l < L; ++l) {
                        const double Hl = (double)shapes[2 * l], Wl = (double)shapes[2 * l + 1];
                        for (int k = 0; k < P; ++k) {
                            const int64_t s = ((int64_t)h * L + l) * P + k;
                            grad_off[(bq * S + s) * 2 + 0] += gl[2 * s + 0] / Wl;
                            grad_off[(bq * S + s) * 2 + 1] += gl[2 * s + 1] / Hl;
                            G[bq * S + s] += ga[s];
                            gr[2 * (k % R) + 0] += gl[2 * s + 0];
                            gr[2 * (k % R) + 1] += gl[2 * s + 1];
                        }
                    }
            }
        }
    const int n = L * P;
    for (int64_t bq = 0; bq < (int64_t)B * Nq; ++bq)
        for (int h = 0; h < H; ++h) {
            const int64_t base = bq * S + (int64_t)h * n;
            oracle_softmax(logits + base, 1, n, alpha);
            double dot = 0.0;
            for (int j = 0; j < n; ++j) dot += alpha[j] * G[base + j];
            for (int j = 0; j < n; ++j) grad_logits[base + j] = alpha[j] * (G[base + j] - dot);
        }
    free(idx); free(count); free(pos); free(hits); free(G); free(alpha);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Temporal Self-Attention ([TS] section 二.2 and the BEV encoder listing)  */
/* ------------------------------------------------------------------------ */

int oracle_tsa_reference_points(int B, int T, int bev_h, int bev_w, double gx, double gy,
                                const double* ego, double* ref)
{
    if (B < 0 || T < 1 || bev_h < 1 || bev_w < 1 || !(gx > 0.0) || !(gy > 0.0) || !ego || !ref)
        return -1;
    const double pi = 3.14159265358979323846;
    const int64_t Nq = (int64_t)bev_h * bev_w;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            const double* e = ego + ((int64_t)b * T + t) * 3;
            const double dx = e[0], dy = e[1], theta = e[2] * pi / 180.0;
            const double cs = cos(theta), sn = sin(theta);
            for (int i = 0; i < bev_h; ++i)
                for (int j = 0; j < bev_w; ++j) {
                    /* cell centre in metres about the BEV centre (x along the width) */
                    const double px = ((double)j + 0.5 - 0.5 * bev_w) * gx;
                    const double py = ((double)i + 0.5 - 0.5 * bev_h) * gy;
                    /* the same point in queue t's frame: rotation, then translation */
                    const double qx = cs * px - sn * py + dx;
                    const double qy = sn * px + cs * py + dy;
                    double* r = ref + (((int64_t)b * T + t) * Nq + (int64_t)i * bev_w + j) * 2;
                    r[0] = qx / (bev_w * gx) + 0.5;
                    r[1] = qy / (bev_h * gy) + 0.5;
                }
        }
    return 0;
}

int oracle_tsa_forward(const double* value, int B, int T, int Nv, int H, int Dh,
                       int L, const int64_t* shapes, const int64_t* starts,
                       int Nq, int P, int R, const double* ref,
                       const double* off, const double* logits,
                       int coord_f32, double* out)
{
    if (T < 1 || B < 0 || out == NULL) return -1;
    const int64_t HD = (int64_t)H * Dh;
    double* per_queue = (double*)malloc(sizeof(double) * (size_t)((int64_t)B * T * Nq * HD + 1));
    if (!per_queue) return -1;
    int rc = oracle_msda_forward_fused(value, B * T, Nv, H, Dh, L, shapes, starts, Nq, P, R, ref,
                                       off, logits, coord_f32, per_queue);
    if (rc == 0)
        for (int b = 0; b < B; ++b)
            for (int q = 0; q < Nq; ++q)
                for (int64_t d = 0; d < HD; ++d) {
                    double sum = 0.0;
                    for (int t = 0; t < T; ++t)
                        sum += per_queue[(((int64_t)b * T + t) * Nq + q) * HD + d];
                    out[((int64_t)b * Nq + q) * HD + d] = sum / T;
                }
    free(per_queue);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Dropout on the module's update branch ([BQ] 12, training time), with the */
/* counter-based generator Philox4x32-10 (Salmon, Moraes, Dror, Shaw,       */
/* "Parallel random numbers: as easy as 1, 2, 3", SC 2011)                 */
/* ------------------------------------------------------------------------ */

void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        /* one Philox S-box round: two 32x32 -> 64-bit products */
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        const uint32_t n1 = (uint32_t)p1;
        const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        const uint32_t n3 = (uint32_t)p0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        /* key schedule: the Weyl increments (golden ratio, sqrt(3) - 1) */
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

int oracle_dropout(const double* o, int64_t n, double p, uint64_t seed, double* out)
{
    if (!o || !out || n < 0 || !(p >= 0.0) || !(p < 1.0)) return -1;
    /* element e keeps its value when word e mod 4 of the generator at counter
     * (e div 4, 0, 0) and key (seed) is at least p * 2^32 */
    const uint64_t thr = (uint64_t)(p * 4294967296.0);
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    for (int64_t e = 0; e < n; ++e) {
        const uint64_t blk = (uint64_t)e >> 2;
        const uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), 0u, 0u};
        uint32_t u[4];
        oracle_philox4x32_10(ctr, key, u);
        out[e] = ((uint64_t)u[e & 3] >= thr) ? o[e] / (1.0 - p) : 0.0;
    }
    return 0;
}
