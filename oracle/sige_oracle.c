/*
 * Plain CPU oracle for SIGE's tile-based sparse convolution.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file; only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * What it computes, and where the pages say so:
 *   - The engine compares the original and edited inputs to get a difference
 *     mask, reuses cached activations outside the edit and re-applies the
 *     filters only on the edit (mer.dev notes on SIGE, section 3 "Method").
 *   - The mask is downsampled to several scales, then dilated, and the
 *     result selects tiles (mer.dev notes, section 3.2 "Sparse Engine SIGE").
 *   - The mask is reduced to active-block indices; active blocks, each with
 *     its halo (overlap 2 for a 3x3 stride-1 conv), are gathered from the
 *     edited activation, stacked on the batch axis and run through F_l; the
 *     output blocks are scattered back into the cached F_l(A_original)
 *     (SIGE project page, "Overview").
 *
 * The oracle writes the plain definition of that result: the layer output
 * equals the cached original output everywhere except at the pixels of the
 * listed tiles, where it equals the layer applied to the edited input.  The
 * layer itself is a direct convolution summed in double precision in a fixed
 * (r, c, ci) order, with zero padding, optional per-channel GroupNorm affine
 * and SiLU on the input, bias and an optional residual.  Readings of points
 * the pages leave open are listed where they are used.
 *
 * Precision: sums in double; the single difference test that turns floats
 * into mask bits is taken in float, the precision the GPU kernel uses for
 * that decision, so that both sides make identical integer decisions.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { O_U8 = 0, O_F32 = 1, O_BF16 = 2 };
enum { O_NHWC = 0, O_NCHW = 1 };

/* ---------------------------------------------------------------- helpers */

static float bf16_bits_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* One stored element widened exactly to float (u8, bf16 and f32 all embed
 * exactly in float). */
static float elem_f(const void *p, int dtype, size_t i)
{
    switch (dtype) {
    case O_U8: return (float)((const uint8_t *)p)[i];
    case O_F32: return ((const float *)p)[i];
    default: return bf16_bits_to_float(((const uint16_t *)p)[i]);
    }
}

static size_t at(int layout, int H, int W, int C, int n, int y, int x, int c)
{
    if (layout == O_NHWC)
        return (((size_t)n * H + y) * W + x) * C + c;
    return (((size_t)n * C + c) * H + y) * W + x;
}

/* Round a double to the nearest bfloat16 (8 significant bits), ties to even,
 * in one step (no intermediate rounding to float).  Returns the bf16 bits. */
uint16_t oracle_round_bf16_one(double d)
{
    if (isnan(d))
        return 0x7FC0;
    uint16_t sign = signbit(d) ? 0x8000 : 0;
    double a = fabs(d);
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e);              /* a = m * 2^e, m in [0.5, 1) -> a in [2^(e-1), 2^e) */
    int q = e - 8;             /* quantum: 8 significant bits */
    if (q < -133)              /* subnormal range of bf16: quantum 2^-133 */
        q = -133;
    double r = nearbyint(ldexp(a, -q)); /* default rounding mode: ties to even */
    double v = ldexp(r, q);
    if (v >= 0x1p128)
        return sign | 0x7F80;  /* overflow to infinity */
    /* v is exactly representable in bf16: take the top 16 bits of its float */
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)((u >> 16) & 0x7FFF);
}

void oracle_round_bf16(const double *in, uint16_t *out, long n)
{
    for (long i = 0; i < n; ++i)
        out[i] = oracle_round_bf16_one(in[i]);
}

static double bf16_roundtrip(double d) { return (double)bf16_bits_to_float(oracle_round_bf16_one(d)); }

/* ------------------------------------------------------ difference mask */

/* Pixel difference mask, OR-ed over the batch:
 *   m[y][x] = OR_n ( max_c |A_edit - A_orig| > threshold ).
 * Reading: maximum over channels of the absolute difference, strict ">", the
 * difference taken in float (u8 inputs differ by an exact integer).  NaN
 * differences never set a bit. */
void oracle_pixel_mask(const void *a_orig, const void *a_edit, int N, int H, int W, int C,
                       int dtype, int layout, float threshold, uint8_t *mask)
{
    for (int y = 0; y < H; ++y)
        for (int x = 0; x < W; ++x) {
            int set = 0;
            for (int n = 0; n < N; ++n) {
                float mx = 0.0f;
                for (int c = 0; c < C; ++c) {
                    size_t i = at(layout, H, W, C, n, y, x, c);
                    float d = fabsf(elem_f(a_edit, dtype, i) - elem_f(a_orig, dtype, i));
                    if (d > mx)
                        mx = d;
                }
                if (mx > threshold)
                    set = 1;
            }
            mask[(size_t)y * W + x] = (uint8_t)set;
        }
}

/* --------------------------------------------- multi-scale index lists */

/* Downsample to (Hs, Ws): a coarse pixel is set when any fine pixel that
 * maps onto it (floor(y*Hs/H) == Y) is set.  Reading: OR-pooling, so an edit
 * is never dropped. */
void oracle_downsample(const uint8_t *m, int H, int W, int Hs, int Ws, uint8_t *ms)
{
    memset(ms, 0, (size_t)Hs * Ws);
    for (int y = 0; y < H; ++y)
        for (int x = 0; x < W; ++x)
            if (m[(size_t)y * W + x])
                ms[(size_t)((long)y * Hs / H) * Ws + (long)x * Ws / W] = 1;
}

/* Dilate by a square of radius R pixels, clipped at the border. */
void oracle_dilate(const uint8_t *ms, int Hs, int Ws, int R, uint8_t *md)
{
    for (int Y = 0; Y < Hs; ++Y)
        for (int X = 0; X < Ws; ++X) {
            int set = 0;
            for (int dy = -R; dy <= R && !set; ++dy)
                for (int dx = -R; dx <= R; ++dx) {
                    int yy = Y + dy, xx = X + dx;
                    if (yy >= 0 && yy < Hs && xx >= 0 && xx < Ws && ms[(size_t)yy * Ws + xx]) {
                        set = 1;
                        break;
                    }
                }
            md[(size_t)Y * Ws + X] = (uint8_t)set;
        }
}

/* One scale: downsample, dilate, tile, list.
 * Reading: the dilation is D tiles, taken as D*b pixels at that scale (a
 * square), before the b x b tiles are formed; a tile is active when any of
 * its pixels is set; tiles are anchored at (0,0) and clipped at the border.
 * The list holds the (row, col) origin of every active tile at that scale,
 * in row-major tile order.  Returns the number of active tiles; writes at
 * most `capacity` pairs. */
int oracle_reduce_scale(const uint8_t *mask, int H, int W, int Hs, int Ws, int b, int D,
                        int32_t *idx, int capacity)
{
    uint8_t *ms = (uint8_t *)malloc((size_t)Hs * Ws);
    uint8_t *md = (uint8_t *)malloc((size_t)Hs * Ws);
    oracle_downsample(mask, H, W, Hs, Ws, ms);
    oracle_dilate(ms, Hs, Ws, D * b, md);
    int th = (Hs + b - 1) / b, tw = (Ws + b - 1) / b, count = 0;
    for (int i = 0; i < th; ++i)
        for (int j = 0; j < tw; ++j) {
            int act = 0;
            for (int y = i * b; y < (i + 1) * b && y < Hs && !act; ++y)
                for (int x = j * b; x < (j + 1) * b && x < Ws; ++x)
                    if (md[(size_t)y * Ws + x]) {
                        act = 1;
                        break;
                    }
            if (act) {
                if (count < capacity) {
                    idx[2 * count] = i * b;
                    idx[2 * count + 1] = j * b;
                }
                ++count;
            }
        }
    free(ms);
    free(md);
    return count;
}

/* ----------------------------------------------------- GroupNorm affine */

/* GroupNorm statistics of the cached ORIGINAL activation, folded into a
 * per-(n, channel) scale and shift: y = x * scale + shift with
 * scale = gamma / sqrt(var + eps), shift = beta - mean * scale.
 * Mean and (biased) variance over H, W and the C/G channels of each group,
 * two passes in double.  Reading: the pages mention no normalisation; taking
 * the statistics from the cached original keeps every op spatially local. */
void oracle_gn_affine(const void *x, int N, int H, int W, int C, int dtype, int groups,
                      const float *gamma, const float *beta, double eps, double *scale,
                      double *shift)
{
    int cg = C / groups;
    for (int n = 0; n < N; ++n)
        for (int g = 0; g < groups; ++g) {
            double cnt = (double)H * W * cg, s = 0.0, v = 0.0;
            for (int y = 0; y < H; ++y)
                for (int xx = 0; xx < W; ++xx)
                    for (int c = g * cg; c < (g + 1) * cg; ++c)
                        s += elem_f(x, dtype, at(O_NHWC, H, W, C, n, y, xx, c));
            double mean = s / cnt;
            for (int y = 0; y < H; ++y)
                for (int xx = 0; xx < W; ++xx)
                    for (int c = g * cg; c < (g + 1) * cg; ++c) {
                        double d = elem_f(x, dtype, at(O_NHWC, H, W, C, n, y, xx, c)) - mean;
                        v += d * d;
                    }
            double var = v / cnt;
            for (int c = g * cg; c < (g + 1) * cg; ++c) {
                double sc = (double)gamma[c] / sqrt(var + eps);
                scale[(size_t)n * C + c] = sc;
                shift[(size_t)n * C + c] = (double)beta[c] - mean * sc;
            }
        }
}

/* --------------------------------------------------------------- layer */

typedef struct {
    int N, H, W, Cin, Cout, k, stride, pad, Ho, Wo, dtype;
} layer_t;

/* Conv input after the optional per-channel transform:
 * t = x * scale + shift, then SiLU t / (1 + exp(-t)) when silu != 0; for
 * bf16 layers the transformed value is rounded to bf16, as the stacked
 * blocks are stored in the layer's dtype.  Computed once per element into a
 * double image (the transform is elementwise, so this is its definition). */
static double *transformed_input(const layer_t *L, const void *x, const double *scale,
                                 const double *shift, int silu)
{
    size_t n = (size_t)L->N * L->H * L->W * L->Cin;
    double *t = (double *)malloc(n * sizeof(double));
#pragma omp parallel for schedule(static)
    for (long i = 0; i < (long)n; ++i) {
        double v = elem_f(x, L->dtype, (size_t)i);
        if (scale) {
            int c = (int)(i % L->Cin);
            int nn = (int)(i / ((size_t)L->H * L->W * L->Cin));
            v = v * scale[(size_t)nn * L->Cin + c] + shift[(size_t)nn * L->Cin + c];
            if (silu)
                v = v / (1.0 + exp(-v));
            if (L->dtype == O_BF16)
                v = bf16_roundtrip(v);
        }
        t[i] = v;
    }
    return t;
}

static double *weights_f64(const layer_t *L, const void *w)
{
    size_t n = (size_t)L->Cout * L->k * L->k * L->Cin;
    double *d = (double *)malloc(n * sizeof(double));
    for (size_t i = 0; i < n; ++i)
        d[i] = elem_f(w, L->dtype, i);
    return d;
}

/* Direct convolution at one output pixel for every output channel:
 *   z[o] = sum_{r,c,ci} W[o][r][c][ci] * X[n][yo*s - p + r][xo*s - p + c][ci]
 * with X = 0 outside the image, then + bias[o] + residual[n][yo][xo][o]. */
static void conv_pixel(const layer_t *L, const double *xt, const double *wd, const float *bias,
                       const void *residual, int n, int yo, int xo, double *z)
{
    for (int o = 0; o < L->Cout; ++o) {
        double acc = 0.0;
        for (int r = 0; r < L->k; ++r) {
            int y = yo * L->stride - L->pad + r;
            if (y < 0 || y >= L->H)
                continue;
            for (int c = 0; c < L->k; ++c) {
                int x = xo * L->stride - L->pad + c;
                if (x < 0 || x >= L->W)
                    continue;
                const double *xp = xt + (((size_t)n * L->H + y) * L->W + x) * L->Cin;
                const double *wp = wd + (((size_t)o * L->k + r) * L->k + c) * L->Cin;
                for (int i = 0; i < L->Cin; ++i)
                    acc += wp[i] * xp[i];
            }
        }
        if (bias)
            acc += (double)bias[o];
        if (residual)
            acc += elem_f(residual, L->dtype, (((size_t)n * L->Ho + yo) * L->Wo + xo) * L->Cout + o);
        z[o] = acc;
    }
}

static void store_out(int dtype, void *y, size_t i, double v)
{
    if (dtype == O_BF16)
        ((uint16_t *)y)[i] = oracle_round_bf16_one(v);
    else
        ((float *)y)[i] = (float)v;
}

static void layer_init(layer_t *L, int N, int H, int W, int Cin, int Cout, int k, int stride, int pad,
                       int dtype)
{
    L->N = N; L->H = H; L->W = W; L->Cin = Cin; L->Cout = Cout; L->k = k; L->stride = stride;
    L->pad = pad; L->dtype = dtype;
    L->Ho = (H + 2 * pad - k) / stride + 1;
    L->Wo = (W + 2 * pad - k) / stride + 1;
}

/* Dense layer, unrounded, in double: z[n][yo][xo][o]. */
void oracle_dense_conv_f64(const void *x, int N, int H, int W, int Cin, int dtype, const void *w,
                           const float *bias, int Cout, int k, int stride, int pad,
                           const double *gn_scale, const double *gn_shift, int silu,
                           const void *residual, double *z)
{
    layer_t L;
    layer_init(&L, N, H, W, Cin, Cout, k, stride, pad, dtype);
    double *xt = transformed_input(&L, x, gn_scale, gn_shift, silu);
    double *wd = weights_f64(&L, w);
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int n = 0; n < N; ++n)
        for (int yo = 0; yo < L.Ho; ++yo)
            for (int xo = 0; xo < L.Wo; ++xo)
                conv_pixel(&L, xt, wd, bias, residual, n, yo, xo,
                           z + (((size_t)n * L.Ho + yo) * L.Wo + xo) * Cout);
    free(xt);
    free(wd);
}

/* Dense layer rounded once to the layer dtype (f32 or bf16). */
void oracle_dense_conv(const void *x, int N, int H, int W, int Cin, int dtype, const void *w,
                       const float *bias, int Cout, int k, int stride, int pad,
                       const double *gn_scale, const double *gn_shift, int silu,
                       const void *residual, void *y)
{
    layer_t L;
    layer_init(&L, N, H, W, Cin, Cout, k, stride, pad, dtype);
    double *xt = transformed_input(&L, x, gn_scale, gn_shift, silu);
    double *wd = weights_f64(&L, w);
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int n = 0; n < N; ++n)
        for (int yo = 0; yo < L.Ho; ++yo) {
            double *z = (double *)malloc(sizeof(double) * Cout);
            for (int xo = 0; xo < L.Wo; ++xo) {
                conv_pixel(&L, xt, wd, bias, residual, n, yo, xo, z);
                for (int o = 0; o < Cout; ++o)
                    store_out(dtype, y, (((size_t)n * L.Ho + yo) * L.Wo + xo) * Cout + o, z[o]);
            }
            free(z);
        }
    free(xt);
    free(wd);
}

/* Sparse layer: y_out = y_cached, then for every listed tile (origin (h0, w0)
 * in output pixels, edge b) and every output pixel of that tile inside the
 * image, y_out = round(layer(x_edit)) at that pixel.  Everything else keeps
 * the cached bytes. */
void oracle_sparse_conv(const void *x_edit, int N, int H, int W, int Cin, int dtype, const void *w,
                        const float *bias, int Cout, int k, int stride, int pad, int block,
                        const int32_t *idx, int count, const double *gn_scale,
                        const double *gn_shift, int silu, const void *residual,
                        const void *y_cached, void *y_out)
{
    layer_t L;
    layer_init(&L, N, H, W, Cin, Cout, k, stride, pad, dtype);
    size_t esz = dtype == O_BF16 ? 2 : 4;
    memcpy(y_out, y_cached, (size_t)N * L.Ho * L.Wo * Cout * esz);
    double *xt = transformed_input(&L, x_edit, gn_scale, gn_shift, silu);
    double *wd = weights_f64(&L, w);
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int n = 0; n < N; ++n)
        for (int t = 0; t < count; ++t) {
            double *z = (double *)malloc(sizeof(double) * Cout);
            int h0 = idx[2 * t], w0 = idx[2 * t + 1];
            for (int i = 0; i < block; ++i)
                for (int j = 0; j < block; ++j) {
                    int yo = h0 + i, xo = w0 + j;
                    if (yo >= L.Ho || xo >= L.Wo)
                        continue;
                    conv_pixel(&L, xt, wd, bias, residual, n, yo, xo, z);
                    for (int o = 0; o < Cout; ++o)
                        store_out(dtype, y_out, (((size_t)n * L.Ho + yo) * L.Wo + xo) * Cout + o, z[o]);
                }
            free(z);
        }
    free(xt);
    free(wd);
}

/* ------------------------------------------- gather / stacked-block conv */

/* Gather: for every listed tile t (output origin (h0, w0)) and batch item n,
 * block[t][n][hh][ww][ci] = X~[n][h0*s - p + hh][w0*s - p + ww][ci] for
 * hh, ww < b_in = (b - 1)*s + k, with X~ the transformed input of the layer
 * (zero outside the image).  Adjacent tiles' blocks overlap by k - s pixels:
 * 2 for a 3x3 stride-1 conv (SIGE project page, "Overview").  Output in double. */
void oracle_gather(const void *x, int N, int H, int W, int Cin, int dtype, int k, int stride, int pad,
                   int block, const int32_t *idx, int count, const double *gn_scale,
                   const double *gn_shift, int silu, double *blocks)
{
    layer_t L;
    layer_init(&L, N, H, W, Cin, Cin, k, stride, pad, dtype);
    double *xt = transformed_input(&L, x, gn_scale, gn_shift, silu);
    int bin = (block - 1) * stride + k;
    for (int t = 0; t < count; ++t)
        for (int n = 0; n < N; ++n)
            for (int hh = 0; hh < bin; ++hh)
                for (int ww = 0; ww < bin; ++ww) {
                    int y = idx[2 * t] * stride - pad + hh, xx = idx[2 * t + 1] * stride - pad + ww;
                    double *dst = blocks + ((((size_t)t * N + n) * bin + hh) * bin + ww) * Cin;
                    for (int c = 0; c < Cin; ++c)
                        dst[c] = (y >= 0 && y < H && xx >= 0 && xx < W)
                                     ? xt[(((size_t)n * H + y) * W + xx) * Cin + c]
                                     : 0.0;
                }
    free(xt);
}

/* Valid convolution of each stacked block (the layer F_l run on the batch of
 * blocks, without bias):
 *   out[m][i][j][o] = sum_{r,c,ci} W[o][r][c][ci] * block[m][i*s + r][j*s + c][ci]
 * for i, j < b.  Blocks in double, output in double. */
void oracle_block_conv(const double *blocks, int nblocks, int Cin, const void *w, int dtype, int Cout,
                       int k, int stride, int block, double *out)
{
    int bin = (block - 1) * stride + k;
    layer_t L;
    layer_init(&L, 1, bin, bin, Cin, Cout, k, stride, 0, dtype);
    double *wd = weights_f64(&L, w);
#pragma omp parallel for schedule(dynamic, 1)
    for (int m = 0; m < nblocks; ++m)
        for (int i = 0; i < block; ++i)
            for (int j = 0; j < block; ++j)
                for (int o = 0; o < Cout; ++o) {
                    double acc = 0.0;
                    for (int r = 0; r < k; ++r)
                        for (int c = 0; c < k; ++c) {
                            const double *bp = blocks + (((size_t)m * bin + i * stride + r) * bin + j * stride + c) * Cin;
                            const double *wp = wd + (((size_t)o * k + r) * k + c) * Cin;
                            for (int ci = 0; ci < Cin; ++ci)
                                acc += wp[ci] * bp[ci];
                        }
                    out[(((size_t)m * block + i) * block + j) * Cout + o] = acc;
                }
    free(wd);
}

/* ------------------------------------------ other layer types (GauGAN) */

/* Transposed convolution (the learned upsampling layer of a generator's
 * decoder; mer.dev notes on SIGE, section 5: GauGAN-style generators beside
 * the plain convs), written in the textbook scatter form: every input pixel
 * (i, j) adds W[o][r][c][ci] * X[n][i][j][ci] to output pixel
 * (i*s - p + r, j*s - p + c), for r, c < k, when that pixel lies in the
 * Ho x Wo output, Ho = (H - 1)*s - 2p + k + op.  The weight is stored
 * [C_out][k][k][C_in] like every other layer here: W[o][r][c][ci] is the
 * coupling of input channel ci to output channel o at tap (r, c).  Optional
 * per-channel affine + SiLU on the input as in the other layers, bias, and a
 * residual of the output's shape.  Sums in double; the scatter visits input
 * pixels row-major and taps (r, c, ci) in order, so each output element is
 * summed in a fixed order. */
static void conv_transpose_f64(const void *x, int N, int H, int W, int Cin, int dtype, const void *w,
                               const float *bias, int Cout, int k, int s, int p, int op, const double *scale,
                               const double *shift, int silu, const void *residual, double *z)
{
    layer_t L;
    layer_init(&L, N, H, W, Cin, Cout, k, 1, 0, dtype);
    int Ho = (H - 1) * s - 2 * p + k + op, Wo = (W - 1) * s - 2 * p + k + op;
    double *xt = transformed_input(&L, x, scale, shift, silu);
    double *wd = weights_f64(&L, w);
    size_t nz = (size_t)N * Ho * Wo * Cout;
    for (size_t i = 0; i < nz; ++i)
        z[i] = 0.0;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n)
        for (int i = 0; i < H; ++i)
            for (int j = 0; j < W; ++j) {
                const double *xp = xt + (((size_t)n * H + i) * W + j) * Cin;
                for (int r = 0; r < k; ++r) {
                    int y = i * s - p + r;
                    if (y < 0 || y >= Ho)
                        continue;
                    for (int c = 0; c < k; ++c) {
                        int xo = j * s - p + c;
                        if (xo < 0 || xo >= Wo)
                            continue;
                        double *zp = z + (((size_t)n * Ho + y) * Wo + xo) * Cout;
                        for (int o = 0; o < Cout; ++o) {
                            const double *wp = wd + (((size_t)o * k + r) * k + c) * Cin;
                            double acc = 0.0;
                            for (int ci = 0; ci < Cin; ++ci)
                                acc += wp[ci] * xp[ci];
                            zp[o] += acc;
                        }
                    }
                }
            }
    for (int n = 0; n < N; ++n)
        for (int y = 0; y < Ho; ++y)
            for (int xo = 0; xo < Wo; ++xo)
                for (int o = 0; o < Cout; ++o) {
                    size_t e = (((size_t)n * Ho + y) * Wo + xo) * Cout + o;
                    if (bias)
                        z[e] += (double)bias[o];
                    if (residual)
                        z[e] += elem_f(residual, dtype, e);
                }
    free(xt);
    free(wd);
}

void oracle_conv_transpose_f64(const void *x, int N, int H, int W, int Cin, int dtype, const void *w,
                               const float *bias, int Cout, int k, int s, int p, int op, const double *scale,
                               const double *shift, int silu, const void *residual, double *z)
{
    conv_transpose_f64(x, N, H, W, Cin, dtype, w, bias, Cout, k, s, p, op, scale, shift, silu, residual, z);
}

/* Tile-masked transposed conv: the cached output, overwritten at the in-image
 * pixels of the listed output tiles (origins in output pixels, edge `block`)
 * by the transposed conv of x_edit rounded once to the dtype. */
void oracle_sparse_conv_transpose(const void *x_edit, int N, int H, int W, int Cin, int dtype, const void *w,
                                  const float *bias, int Cout, int k, int s, int p, int op, int block,
                                  const int32_t *idx, int count, const double *scale, const double *shift,
                                  int silu, const void *residual, const void *y_cached, void *y_out)
{
    int Ho = (H - 1) * s - 2 * p + k + op, Wo = (W - 1) * s - 2 * p + k + op;
    size_t nz = (size_t)N * Ho * Wo * Cout;
    size_t esz = dtype == O_BF16 ? 2 : 4;
    double *z = (double *)malloc(nz * sizeof(double));
    conv_transpose_f64(x_edit, N, H, W, Cin, dtype, w, bias, Cout, k, s, p, op, scale, shift, silu, residual, z);
    memcpy(y_out, y_cached, nz * esz);
    for (int n = 0; n < N; ++n)
        for (int t = 0; t < count; ++t)
            for (int i = 0; i < block; ++i)
                for (int j = 0; j < block; ++j) {
                    int y = idx[2 * t] + i, xo = idx[2 * t + 1] + j;
                    if (y >= Ho || xo >= Wo)
                        continue;
                    for (int o = 0; o < Cout; ++o) {
                        size_t e = (((size_t)n * Ho + y) * Wo + xo) * Cout + o;
                        store_out(dtype, y_out, e, z[e]);
                    }
                }
    free(z);
}

/* SPADE-style input of a GauGAN layer: a parameter-free normalisation whose
 * per-channel statistics are folded into scale/shift (taken, like GroupNorm
 * here, from the cached original activation), then modulated per pixel by
 * maps the generator computes from the segmentation:
 *   t = act((x * scale[n][c] + shift[n][c]) * (1 + gamma[n][y][x][c]) + beta[n][y][x][c])
 * with act = identity (0), SiLU (1) or LeakyReLU with slope 0.2 (2), rounded
 * to bf16 for bf16 layers (the stacked blocks' storage); gamma and beta are
 * NHWC maps of x's shape and dtype.  The conv that follows is the plain
 * direct conv above. */
static double *spade_input(const layer_t *L, const void *x, const double *scale, const double *shift,
                           const void *gamma, const void *beta, int act)
{
    size_t n = (size_t)L->N * L->H * L->W * L->Cin;
    double *t = (double *)malloc(n * sizeof(double));
#pragma omp parallel for schedule(static)
    for (long i = 0; i < (long)n; ++i) {
        int c = (int)(i % L->Cin);
        int nn = (int)(i / ((size_t)L->H * L->W * L->Cin));
        double v = elem_f(x, L->dtype, (size_t)i);
        v = v * scale[(size_t)nn * L->Cin + c] + shift[(size_t)nn * L->Cin + c];
        v = v * (1.0 + elem_f(gamma, L->dtype, (size_t)i)) + elem_f(beta, L->dtype, (size_t)i);
        if (act == 1)
            v = v / (1.0 + exp(-v));
        else if (act == 2)
            v = v >= 0.0 ? v : 0.2 * v;
        if (L->dtype == O_BF16)
            v = bf16_roundtrip(v);
        t[i] = v;
    }
    return t;
}

/* Dense conv of the SPADE input, unrounded (z) or, when y != NULL, rounded
 * once into y; and its tile-masked form when idx != NULL (y_out = y_cached
 * except at the listed tiles). */
void oracle_spade_conv(const void *x, int N, int H, int W, int Cin, int dtype, const void *w, const float *bias,
                       int Cout, int k, int stride, int pad, const double *scale, const double *shift,
                       const void *gamma, const void *beta, int act, const void *residual, int block,
                       const int32_t *idx, int count, const void *y_cached, double *z, void *y_out)
{
    layer_t L;
    layer_init(&L, N, H, W, Cin, Cout, k, stride, pad, dtype);
    double *xt = spade_input(&L, x, scale, shift, gamma, beta, act);
    double *wd = weights_f64(&L, w);
    size_t esz = dtype == O_BF16 ? 2 : 4;
    if (idx && y_out)
        memcpy(y_out, y_cached, (size_t)N * L.Ho * L.Wo * Cout * esz);
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int n = 0; n < N; ++n)
        for (int yo = 0; yo < L.Ho; ++yo) {
            double *acc = (double *)malloc(sizeof(double) * Cout);
            for (int xo = 0; xo < L.Wo; ++xo) {
                int listed = 1;
                if (idx) {
                    listed = 0;
                    for (int t = 0; t < count && !listed; ++t)
                        listed = yo >= idx[2 * t] && yo < idx[2 * t] + block && xo >= idx[2 * t + 1] &&
                                 xo < idx[2 * t + 1] + block;
                }
                if (!listed)
                    continue;
                conv_pixel(&L, xt, wd, bias, residual, n, yo, xo, acc);
                size_t e0 = (((size_t)n * L.Ho + yo) * L.Wo + xo) * Cout;
                for (int o = 0; o < Cout; ++o) {
                    if (z)
                        z[e0 + o] = acc[o];
                    if (y_out)
                        store_out(dtype, y_out, e0 + o, acc[o]);
                }
            }
            free(acc);
        }
    free(xt);
    free(wd);
}
