/*
 * msda_oracle.c -- float64 CPU oracle for the multi-scale deformable attention
 * core (MSDeformAttn): forward and training backward.
 *
 * TEST INFRASTRUCTURE.  This file is the slow, obviously correct statement of
 * what the CUDA path must compute.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load it.  It shares no code,
 * header, table or helper with the CUDA library, and it includes nothing from it.
 *
 * Sources (web pages, cited by title and section):
 *  [notes]  "Deformable DETR Deformable Transformers for End-to-End Object
 *           Detection" (phdsky.com paper notes), 核心洞察 2, the multi-scale
 *           deformable attention equation: for each query and head, the sum over
 *           levels l and points k of A_{mlqk} times the level-l feature sampled at
 *           phi_l(p_q) + dp_{mlqk}; the weights are normalised over the L*K points.
 *  [walk]   "Deformable DETR模型解读（附源码+论文）" (xdnf.cn), encoder walkthrough:
 *           MultiScaleDeformableAttention.forward (value viewed as [N, S, M, D];
 *           locations are reference point + offset / (W_l, H_l), so component 0
 *           goes with the width and component 1 with the height) and
 *           ms_deform_attn_core_pytorch (value split per level, each level a
 *           row-major H_l x W_l map; grid = 2*loc - 1 sampled bilinearly with
 *           zeros padding and align_corners=False; output laid out [N, Lq, M*D]
 *           with channel m*D + d).
 *
 * Readings taken where the pages are silent:
 *  - grid_sample with align_corners=False maps a grid value g in [-1, 1] to the
 *    pixel coordinate ((g + 1) * W - 1) / 2; with g = 2*loc - 1 that is
 *    loc * W - 0.5.  Pixel centres sit at integer coordinates.
 *  - Each of the four bilinear corners is used only if it lies inside the map;
 *    a corner outside contributes zero (zeros padding).  A location whose
 *    coordinate is not finite has no corner inside the map, but its bilinear
 *    weights are NaN: its sample -- and with it the output, grad_attn and
 *    grad_loc of that point -- is NaN, and grad_value receives nothing from it
 *    (this is also what grid_sample does).
 *  - The pages print no backward.  The backward is the exact derivative of the
 *    forward above, taken inside the cell [x0, x0 + 1) x [y0, y0 + 1) with
 *    x0 = floor(x), y0 = floor(y) (the one-sided derivative at integer
 *    coordinates).  attention_weights are inputs: the softmax that produced
 *    them is not differentiated here.
 *
 * Layouts (all row-major, contiguous):
 *   value               [B, S, M, D]        S = sum_l H_l * W_l
 *   spatial_shapes      [L, 2]              row l = (H_l, W_l)
 *   level_start_index   [L]                 first flat token of level l
 *   sampling_locations  [B, Lq, M, L, K, 2] (x, y), normalised
 *   attention_weights   [B, Lq, M, L, K]
 *   output              [B, Lq, M * D]
 *
 * Return value of every entry point: 0 on success, -1 if a shape is negative
 * (or, for the fused entry points, R is neither 2 nor 4), -2 if scratch memory
 * could not be allocated.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

/* Integer pixel coordinate of a corner, or -1 if the corner lies outside [0, n). */
static int64_t corner_index(double c, int64_t n)
{
    if (c >= 0.0 && c <= (double)(n - 1))
        return (int64_t)c;
    return -1;
}

/* The value element behind one corner, zero when the corner is outside the map. */
static double corner_value(const double *value, int64_t S, int64_t M, int64_t D,
                           int64_t b, int64_t start, int64_t W, int64_t xi,
                           int64_t yi, int64_t m, int64_t d)
{
    if (xi < 0 || yi < 0)
        return 0.0;
    return value[((b * S + start + yi * W + xi) * M + m) * D + d];
}

/* One sampling point, mapped to pixels: the cell's corner coordinates and the
 * fractional position inside the cell. */
typedef struct {
    int64_t xi[2]; /* x0, x0 + 1 as indices, -1 where outside */
    int64_t yi[2]; /* y0, y0 + 1 as indices, -1 where outside */
    double fx, fy; /* x - x0, y - y0 */
} cell;

static cell locate(double loc_x, double loc_y, int64_t H, int64_t W)
{
    cell c;
    double x = loc_x * (double)W - 0.5;
    double y = loc_y * (double)H - 0.5;
    double x0 = floor(x);
    double y0 = floor(y);
    c.fx = x - x0;
    c.fy = y - y0;
    c.xi[0] = corner_index(x0, W);
    c.xi[1] = corner_index(x0 + 1.0, W);
    c.yi[0] = corner_index(y0, H);
    c.yi[1] = corner_index(y0 + 1.0, H);
    return c;
}

int msda_oracle_forward(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq,
                        int64_t L, int64_t K, const double *value,
                        const int64_t *spatial_shapes,
                        const int64_t *level_start_index,
                        const double *sampling_locations,
                        const double *attention_weights, double *output)
{
    if (B < 0 || S < 0 || M < 0 || D < 0 || Lq < 0 || L < 0 || K < 0)
        return -1;
    for (int64_t i = 0; i < B * Lq * M * D; ++i)
        output[i] = 0.0;

    for (int64_t b = 0; b < B; ++b)
    for (int64_t q = 0; q < Lq; ++q)
    for (int64_t m = 0; m < M; ++m)
    for (int64_t l = 0; l < L; ++l) {
        int64_t H = spatial_shapes[2 * l + 0];
        int64_t W = spatial_shapes[2 * l + 1];
        int64_t start = level_start_index[l];
        for (int64_t k = 0; k < K; ++k) {
            int64_t p = (((b * Lq + q) * M + m) * L + l) * K + k;
            double A = attention_weights[p];
            cell c = locate(sampling_locations[2 * p + 0],
                            sampling_locations[2 * p + 1], H, W);
            double wx[2] = {1.0 - c.fx, c.fx};
            double wy[2] = {1.0 - c.fy, c.fy};
            for (int64_t d = 0; d < D; ++d) {
                double sample = 0.0;
                for (int j = 0; j < 2; ++j)
                    for (int i = 0; i < 2; ++i)
                        sample += wx[i] * wy[j] *
                                  corner_value(value, S, M, D, b, start, W,
                                               c.xi[i], c.yi[j], m, d);
                output[(b * Lq + q) * M * D + m * D + d] += A * sample;
            }
        }
    }
    return 0;
}

int msda_oracle_backward(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq,
                         int64_t L, int64_t K, const double *value,
                         const int64_t *spatial_shapes,
                         const int64_t *level_start_index,
                         const double *sampling_locations,
                         const double *attention_weights,
                         const double *grad_output, double *grad_value,
                         double *grad_sampling_locations,
                         double *grad_attention_weights)
{
    if (B < 0 || S < 0 || M < 0 || D < 0 || Lq < 0 || L < 0 || K < 0)
        return -1;
    for (int64_t i = 0; i < B * S * M * D; ++i)
        grad_value[i] = 0.0;

    for (int64_t b = 0; b < B; ++b)
    for (int64_t q = 0; q < Lq; ++q)
    for (int64_t m = 0; m < M; ++m)
    for (int64_t l = 0; l < L; ++l) {
        int64_t H = spatial_shapes[2 * l + 0];
        int64_t W = spatial_shapes[2 * l + 1];
        int64_t start = level_start_index[l];
        for (int64_t k = 0; k < K; ++k) {
            int64_t p = (((b * Lq + q) * M + m) * L + l) * K + k;
            double A = attention_weights[p];
            cell c = locate(sampling_locations[2 * p + 0],
                            sampling_locations[2 * p + 1], H, W);
            double wx[2] = {1.0 - c.fx, c.fx};
            double wy[2] = {1.0 - c.fy, c.fy};
            double g_attn = 0.0; /* sum_d gO * sample            */
            double g_x = 0.0;    /* sum_d gO * d(sample)/dx       */
            double g_y = 0.0;    /* sum_d gO * d(sample)/dy       */
            for (int64_t d = 0; d < D; ++d) {
                double gO = grad_output[(b * Lq + q) * M * D + m * D + d];
                double v[2][2]; /* v[j][i] = V(x0 + i, y0 + j) */
                for (int j = 0; j < 2; ++j)
                    for (int i = 0; i < 2; ++i)
                        v[j][i] = corner_value(value, S, M, D, b, start, W,
                                               c.xi[i], c.yi[j], m, d);
                double sample = 0.0;
                for (int j = 0; j < 2; ++j)
                    for (int i = 0; i < 2; ++i)
                        sample += wx[i] * wy[j] * v[j][i];
                g_attn += gO * sample;
                /* d/dx of wx = (1 - fx, fx) is (-1, +1); likewise for y. */
                g_x += gO * (wy[0] * (v[0][1] - v[0][0]) + wy[1] * (v[1][1] - v[1][0]));
                g_y += gO * (wx[0] * (v[1][0] - v[0][0]) + wx[1] * (v[1][1] - v[0][1]));
                for (int j = 0; j < 2; ++j)
                    for (int i = 0; i < 2; ++i)
                        if (c.xi[i] >= 0 && c.yi[j] >= 0)
                            grad_value[((b * S + start + c.yi[j] * W + c.xi[i]) * M + m) * D + d] +=
                                A * wx[i] * wy[j] * gO;
            }
            grad_attention_weights[p] = g_attn;
            /* x = loc_x * W - 0.5, so dx/dloc_x = W; likewise dy/dloc_y = H. */
            grad_sampling_locations[2 * p + 0] = A * (double)W * g_x;
            grad_sampling_locations[2 * p + 1] = A * (double)H * g_y;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * The step before the core: sampling locations and attention weights formed
 * from the raw inputs, then the core above.
 *
 * Sources (same pages): [walk] MultiScaleDeformableAttention.forward and the
 * Deformable DETR MSDeformAttn.forward printed on "Deformable DETR模型解读
 * （附源码+论文）" and on the phdsky.com notes:
 *  - attention weights: a softmax over the L*K logits of each (b, q, m);
 *  - reference points with 2 components (x, y): loc = ref + off / (W_l, H_l);
 *  - reference points with 4 components (box centre x, y and size w, h):
 *    loc = ref[0:2] + off / K * ref[2:4] * 0.5.
 * Readings taken where the pages are silent:
 *  - with round_f32 = 1 the location is formed in float32, every operation
 *    rounded once in the pages' order (division by the normaliser, then the
 *    addition; for boxes the division by K, the product with the size, the
 *    product with 0.5, then the addition), as the pages' float32 tensors
 *    compute it; with round_f32 = 0 it is formed in float64 (used by the
 *    finite-difference checks).  The softmax is float64 either way.
 *  - the backward differentiates the real-number formula (the float32
 *    rounding is not differentiated): d loc / d off = 1 / (W_l, H_l), or
 *    ref[2:4] * 0.5 / K for boxes; d loc / d ref[0:2] = 1; for boxes
 *    d loc / d ref[2:4] = off * 0.5 / K; the softmax gives
 *    d z_i = A_i * (gA_i - sum_j A_j gA_j) over the (b, q, m) group.
 *
 * Extra layouts:
 *   reference_points    [B, Lq, L, R]          R = 2 or 4
 *   sampling_offsets    [B, Lq, M, L, K, 2]
 *   attention_logits    [B, Lq, M, L * K]
 * ------------------------------------------------------------------------ */

static double form_location(double ref_c, double size_c, double off_c, int64_t n,
                            int64_t K, int64_t R, int round_f32)
{
    if (round_f32) {
        float t;
        if (R == 2) {
            t = (float)off_c / (float)n;
        } else {
            t = (float)off_c / (float)K;
            t = t * (float)size_c;
            t = t * 0.5f;
        }
        return (double)((float)ref_c + t);
    }
    if (R == 2)
        return ref_c + off_c / (double)n;
    return ref_c + off_c / (double)K * size_c * 0.5;
}

/* loc [B, Lq, M, L, K, 2] and A [B, Lq, M, L, K] from the raw inputs. */
static void fused_inputs(int64_t B, int64_t Lq, int64_t M, int64_t L, int64_t K,
                         int64_t R, int round_f32, const int64_t *spatial_shapes,
                         const double *ref, const double *off, const double *logits,
                         double *loc, double *A)
{
    int64_t LK = L * K;
    for (int64_t b = 0; b < B; ++b)
    for (int64_t q = 0; q < Lq; ++q)
    for (int64_t m = 0; m < M; ++m) {
        int64_t g = (b * Lq + q) * M + m;
        const double *z = logits + g * LK;
        double zmax = z[0];
        for (int64_t i = 1; i < LK; ++i)
            if (z[i] > zmax || isnan(z[i]))
                zmax = z[i];
        double sum = 0.0;
        for (int64_t i = 0; i < LK; ++i)
            sum += exp(z[i] - zmax);
        for (int64_t i = 0; i < LK; ++i)
            A[g * LK + i] = exp(z[i] - zmax) / sum;
        for (int64_t l = 0; l < L; ++l) {
            const double *r = ref + ((b * Lq + q) * L + l) * R;
            int64_t H = spatial_shapes[2 * l + 0];
            int64_t W = spatial_shapes[2 * l + 1];
            for (int64_t k = 0; k < K; ++k) {
                int64_t p = g * LK + l * K + k;
                loc[2 * p + 0] = form_location(r[0], R == 4 ? r[2] : 0.0, off[2 * p + 0], W,
                                               K, R, round_f32);
                loc[2 * p + 1] = form_location(r[1], R == 4 ? r[3] : 0.0, off[2 * p + 1], H,
                                               K, R, round_f32);
            }
        }
    }
}

int msda_oracle_fused_forward(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq,
                              int64_t L, int64_t K, int64_t R, int round_f32,
                              const double *value, const int64_t *spatial_shapes,
                              const int64_t *level_start_index,
                              const double *reference_points,
                              const double *sampling_offsets,
                              const double *attention_logits, double *output)
{
    if (B < 0 || S < 0 || M < 0 || D < 0 || Lq < 0 || L < 0 || K < 0 || (R != 2 && R != 4))
        return -1;
    int64_t n = B * Lq * M * L * K;
    double *loc = malloc(sizeof(double) * (size_t)(2 * n + 1));
    double *A = malloc(sizeof(double) * (size_t)(n + 1));
    if (loc == NULL || A == NULL) {
        free(loc);
        free(A);
        return -2;
    }
    fused_inputs(B, Lq, M, L, K, R, round_f32, spatial_shapes, reference_points,
                 sampling_offsets, attention_logits, loc, A);
    int rc = msda_oracle_forward(B, S, M, D, Lq, L, K, value, spatial_shapes,
                                 level_start_index, loc, A, output);
    free(loc);
    free(A);
    return rc;
}

int msda_oracle_fused_backward(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq,
                               int64_t L, int64_t K, int64_t R, int round_f32,
                               const double *value, const int64_t *spatial_shapes,
                               const int64_t *level_start_index,
                               const double *reference_points,
                               const double *sampling_offsets,
                               const double *attention_logits, const double *grad_output,
                               double *grad_value, double *grad_sampling_offsets,
                               double *grad_attention_logits,
                               double *grad_reference_points)
{
    if (B < 0 || S < 0 || M < 0 || D < 0 || Lq < 0 || L < 0 || K < 0 || (R != 2 && R != 4))
        return -1;
    int64_t n = B * Lq * M * L * K;
    int64_t LK = L * K;
    double *loc = malloc(sizeof(double) * (size_t)(2 * n + 1));
    double *A = malloc(sizeof(double) * (size_t)(n + 1));
    double *gloc = malloc(sizeof(double) * (size_t)(2 * n + 1));
    double *gA = malloc(sizeof(double) * (size_t)(n + 1));
    if (loc == NULL || A == NULL || gloc == NULL || gA == NULL) {
        free(loc);
        free(A);
        free(gloc);
        free(gA);
        return -2;
    }
    fused_inputs(B, Lq, M, L, K, R, round_f32, spatial_shapes, reference_points,
                 sampling_offsets, attention_logits, loc, A);
    int rc = msda_oracle_backward(B, S, M, D, Lq, L, K, value, spatial_shapes,
                                  level_start_index, loc, A, grad_output, grad_value,
                                  gloc, gA);
    if (rc == 0) {
        if (grad_reference_points != NULL)
            for (int64_t i = 0; i < B * Lq * L * R; ++i)
                grad_reference_points[i] = 0.0;
        for (int64_t b = 0; b < B; ++b)
        for (int64_t q = 0; q < Lq; ++q)
        for (int64_t m = 0; m < M; ++m) {
            int64_t g = (b * Lq + q) * M + m;
            /* Softmax: d z_i = A_i (gA_i - sum_j A_j gA_j). */
            double s = 0.0;
            for (int64_t i = 0; i < LK; ++i)
                s += A[g * LK + i] * gA[g * LK + i];
            for (int64_t i = 0; i < LK; ++i)
                grad_attention_logits[g * LK + i] = A[g * LK + i] * (gA[g * LK + i] - s);
            for (int64_t l = 0; l < L; ++l) {
                const double *r = reference_points + ((b * Lq + q) * L + l) * R;
                double *gr = grad_reference_points == NULL
                                 ? NULL
                                 : grad_reference_points + ((b * Lq + q) * L + l) * R;
                int64_t H = spatial_shapes[2 * l + 0];
                int64_t W = spatial_shapes[2 * l + 1];
                for (int64_t k = 0; k < K; ++k) {
                    int64_t p = g * LK + l * K + k;
                    for (int c = 0; c < 2; ++c) {
                        double gl = gloc[2 * p + c];
                        double dloc_doff = R == 2 ? 1.0 / (double)(c == 0 ? W : H)
                                                  : r[2 + c] * 0.5 / (double)K;
                        grad_sampling_offsets[2 * p + c] = gl * dloc_doff;
                        if (gr != NULL) {
                            gr[c] += gl;
                            if (R == 4)
                                gr[2 + c] += gl * sampling_offsets[2 * p + c] * 0.5 / (double)K;
                        }
                    }
                }
            }
        }
    }
    free(loc);
    free(A);
    free(gloc);
    free(gA);
    return rc;
}
