/*
 * DCNv4 forward spatial aggregation -- plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link or
 * call this file; it exists so that the tests, the smoke check and the CPU
 * baseline of the benchmark have an obviously correct, independent statement
 * of what the operator computes. It shares no code, header, table or helper
 * with the CUDA library.
 *
 * What it computes (sources, by page title and section):
 *  - "不只是卷积的平替：我把DCNv4塞进Stable Diffusion的U-Net里" (jsqmd.com),
 *    section 1: the softmax over the aggregation weights is removed, so the
 *    modulation scalars are used raw and may be negative or exceed 1; the
 *    simplified forward listing of the same section adds learned offsets,
 *    reshaped as (N, G, 2, K*K, H, W), to a regular K x K grid, bilinearly
 *    samples the input there, weights every sample by its mask value and sums
 *    over the K*K axis, group by group.
 *  - "掌握DCNv4技术：3倍速度提升与80%加速效果的实战指南" (pwwt.cn), tuning
 *    section: offset_scale multiplies the offsets.
 *  - Operator contract of this library: channels-last x[N,H,W,C], packed
 *    offset_mask[N,Hout,Wout,G,3*K*K] with, per group, 2*K*K offsets then
 *    K*K masks, zero padding outside the image, out[N,Hout,Wout,C].
 *
 * Readings taken where the pages are silent:
 *  - grid point order is row-major, k = ky*K + kx;
 *  - the grid is convolution style: p0 = o*stride - pad + kk*dilation;
 *  - offsets are component-major inside the 2*K*K block: r[k] moves along
 *    the width (x), r[K*K + k] along the height (y); masks are r[2*K*K + k];
 *  - the scaled offset is one fp32 multiply, fl32(offset_scale * r), which is
 *    exact when offset_scale == 1; the sample position is p0 + that value;
 *  - zero padding is per corner: corners outside the image contribute 0,
 *    corners inside always contribute (even with weight 0); a non-finite
 *    offset puts the whole sample outside;
 *  - offsets are in pixels.
 *
 * Precision: inputs arrive as fp64 copies of the (already rounded) storage
 * values; everything else is fp64 except the single fp32 offset multiply.
 * Compile with -ffp-contract=off so that no multiply-add is fused.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Output extent of one spatial axis, convolution style. Returns <= 0 when no
 * output position exists. */
int oracle_output_size(int in, int K, int stride, int pad, int dilation)
{
    long span = (long)in + 2L * pad - (long)dilation * (K - 1) - 1;
    if (stride <= 0 || span < 0) return 0;
    return (int)(span / stride + 1);
}

/* The scaled offset: fl32(offset_scale * r). r holds a value that is exactly
 * representable in fp32 (it came from fp32, fp16 or bf16 storage). */
static double scaled_offset(float offset_scale, double r)
{
    volatile float prod = offset_scale * (float)r; /* one fp32 rounding */
    return (double)prod;
}

/* One output element group: out[n, ho, wo, g*Cg : (g+1)*Cg].
 * Sums over the K*K grid points of group g the bilinear sample of x at
 * p0 + offset, weighted by the raw mask value. */
static void aggregate_one(const double *x, const double *om, double *out,
                          int N, int H, int W, int C, int G, int K,
                          int stride, int pad, int dilation, float offset_scale,
                          int Hout, int Wout, int n, int ho, int wo, int g)
{
    const int Cg = C / G;
    const int KK = K * K;
    const double *r = om + ((((size_t)n * Hout + ho) * Wout + wo) * G + g) * (size_t)(3 * KK);
    double *o = out + (((size_t)n * Hout + ho) * Wout + wo) * (size_t)C + (size_t)g * Cg;
    (void)N;

    for (int c = 0; c < Cg; ++c) o[c] = 0.0;

    for (int k = 0; k < KK; ++k) {
        const int ky = k / K, kx = k % K;
        const int p0y = ho * stride - pad + ky * dilation;
        const int p0x = wo * stride - pad + kx * dilation;
        const double dx = scaled_offset(offset_scale, r[k]);
        const double dy = scaled_offset(offset_scale, r[KK + k]);
        const double m = r[2 * KK + k];
        if (!isfinite(dx) || !isfinite(dy)) continue; /* outside the image */

        /* sample position (p0y + dy, p0x + dx); its top-left corner and the
         * fractional part, without rounding p0 + d */
        const double fy0 = floor(dy), fx0 = floor(dx);
        const double ly = dy - fy0, lx = dx - fx0;
        const double y0 = (double)p0y + fy0, x0 = (double)p0x + fx0;

        for (int a = 0; a <= 1; ++a) {
            for (int b = 0; b <= 1; ++b) {
                const double yy = y0 + a, xx = x0 + b;
                if (!(yy >= 0.0 && yy <= (double)(H - 1) && xx >= 0.0 && xx <= (double)(W - 1)))
                    continue; /* zero padding */
                const double wy = a ? ly : 1.0 - ly;
                const double wx = b ? lx : 1.0 - lx;
                const double w = m * wy * wx;
                const double *px = x + ((((size_t)n * H + (size_t)yy) * W + (size_t)xx) * C) + (size_t)g * Cg;
                for (int c = 0; c < Cg; ++c) o[c] += w * px[c];
            }
        }
    }
}

/* Full forward. x: [N,H,W,C]; om: [N,Hout,Wout,G,3*K*K]; out: [N,Hout,Wout,C].
 * All fp64, contiguous. Returns 0, or -1 on inconsistent arguments. */
int oracle_dcnv4_forward(const double *x, const double *om, double *out,
                         int N, int H, int W, int C, int G, int K,
                         int stride, int pad, int dilation, float offset_scale)
{
    if (N < 0 || H <= 0 || W <= 0 || C <= 0 || G <= 0 || K <= 0 || C % G) return -1;
    const int Hout = oracle_output_size(H, K, stride, pad, dilation);
    const int Wout = oracle_output_size(W, K, stride, pad, dilation);
    if (Hout <= 0 || Wout <= 0) return -1;
    for (int n = 0; n < N; ++n)
        for (int ho = 0; ho < Hout; ++ho)
            for (int wo = 0; wo < Wout; ++wo)
                for (int g = 0; g < G; ++g)
                    aggregate_one(x, om, out, N, H, W, C, G, K, stride, pad, dilation,
                                  offset_scale, Hout, Wout, n, ho, wo, g);
    return 0;
}

/* Same as oracle_dcnv4_forward restricted to images [n_begin, n_end): used to
 * time a bounded sample of a large workload. Pointers address the full
 * tensors. */
int oracle_dcnv4_forward_images(const double *x, const double *om, double *out,
                                int N, int H, int W, int C, int G, int K,
                                int stride, int pad, int dilation, float offset_scale,
                                int n_begin, int n_end)
{
    if (n_begin < 0 || n_end > N || n_begin > n_end || C % G) return -1;
    const int Hout = oracle_output_size(H, K, stride, pad, dilation);
    const int Wout = oracle_output_size(W, K, stride, pad, dilation);
    if (Hout <= 0 || Wout <= 0) return -1;
    for (int n = n_begin; n < n_end; ++n)
        for (int ho = 0; ho < Hout; ++ho)
            for (int wo = 0; wo < Wout; ++wo)
                for (int g = 0; g < G; ++g)
                    aggregate_one(x, om, out, N, H, W, C, G, K, stride, pad, dilation,
                                  offset_scale, Hout, Wout, n, ho, wo, g);
    return 0;
}

/* oracle_dcnv4_forward_images with the (image, output row) pairs shared out
 * among `threads` OpenMP threads (threads <= 0: the OpenMP default). Every
 * output element is still computed by aggregate_one, alone and in the same
 * order, so the result is bit-identical to the single-thread call; only the
 * wall time changes. Used to time the oracle on all host cores. */
int oracle_dcnv4_forward_images_mt(const double *x, const double *om, double *out,
                                   int N, int H, int W, int C, int G, int K,
                                   int stride, int pad, int dilation, float offset_scale,
                                   int n_begin, int n_end, int threads)
{
    if (n_begin < 0 || n_end > N || n_begin > n_end || C % G) return -1;
    const int Hout = oracle_output_size(H, K, stride, pad, dilation);
    const int Wout = oracle_output_size(W, K, stride, pad, dilation);
    if (Hout <= 0 || Wout <= 0) return -1;
    const long rows = (long)(n_end - n_begin) * Hout;
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#else
    (void)threads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (long r = 0; r < rows; ++r) {
        const int n = n_begin + (int)(r / Hout), ho = (int)(r % Hout);
        for (int wo = 0; wo < Wout; ++wo)
            for (int g = 0; g < G; ++g)
                aggregate_one(x, om, out, N, H, W, C, G, K, stride, pad, dilation,
                              offset_scale, Hout, Wout, n, ho, wo, g);
    }
    return 0;
}

/* Number of threads an OpenMP parallel region of this library would use
 * (1 when it is built without OpenMP). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Integer part of every sample: the top-left corner (y0, x0) and a 4-bit mask
 * of the corners that lie inside the image (bit 0: (y0,x0), bit 1: (y0,x0+1),
 * bit 2: (y0+1,x0), bit 3: (y0+1,x0+1)).
 * corner: [N,Hout,Wout,G,K*K,2] int32 (y0 then x0); valid: [N,Hout,Wout,G,K*K].
 * A sample with no corner inside reports corner = (INT32_MIN, INT32_MIN). */
int oracle_dcnv4_sampling_index(const double *om, int32_t *corner, uint8_t *valid,
                                int N, int H, int W, int G, int K,
                                int stride, int pad, int dilation, float offset_scale)
{
    const int Hout = oracle_output_size(H, K, stride, pad, dilation);
    const int Wout = oracle_output_size(W, K, stride, pad, dilation);
    if (Hout <= 0 || Wout <= 0 || G <= 0 || K <= 0) return -1;
    const int KK = K * K;
    for (int n = 0; n < N; ++n)
        for (int ho = 0; ho < Hout; ++ho)
            for (int wo = 0; wo < Wout; ++wo)
                for (int g = 0; g < G; ++g) {
                    const size_t unit = (((size_t)n * Hout + ho) * Wout + wo) * G + g;
                    const double *r = om + unit * (size_t)(3 * KK);
                    for (int k = 0; k < KK; ++k) {
                        const int ky = k / K, kx = k % K;
                        const int p0y = ho * stride - pad + ky * dilation;
                        const int p0x = wo * stride - pad + kx * dilation;
                        const double dx = scaled_offset(offset_scale, r[k]);
                        const double dy = scaled_offset(offset_scale, r[KK + k]);
                        unsigned bits = 0;
                        double y0 = 0, x0 = 0;
                        if (isfinite(dx) && isfinite(dy)) {
                            y0 = (double)p0y + floor(dy);
                            x0 = (double)p0x + floor(dx);
                            for (int a = 0; a <= 1; ++a)
                                for (int b = 0; b <= 1; ++b) {
                                    const double yy = y0 + a, xx = x0 + b;
                                    if (yy >= 0.0 && yy <= (double)(H - 1) &&
                                        xx >= 0.0 && xx <= (double)(W - 1))
                                        bits |= 1u << (2 * a + b);
                                }
                        }
                        const size_t p = unit * KK + k;
                        valid[p] = (uint8_t)bits;
                        corner[2 * p + 0] = bits ? (int32_t)y0 : INT32_MIN;
                        corner[2 * p + 1] = bits ? (int32_t)x0 : INT32_MIN;
                    }
                }
    return 0;
}

/* ------------------------------------------------------------------------
 * Variants of the forward. "掌握DCNv4技术" (pwwt.cn), section on advanced
 * tuning and extension: DCNv4 also offers centre feature scaling (a sigmoid
 * that weighs the feature at the centre against the aggregate) and the
 * removal of the centre point. "不只是卷积的平替" (jsqmd.com), section 1:
 * DCNv3 normalised the K*K aggregation weights with a softmax, which DCNv4
 * drops; the flag below restores it for comparison.
 *
 * Readings taken here (the pages give no formulas):
 *  - softmax: per (n, ho, wo, g), m'_j = exp(m_j - max) / sum_i exp(m_i - max)
 *    over the unit's points, then the aggregation of the forward with m';
 *  - remove_center (K odd, K >= 3): the unit has P = K*K - 1 points, its
 *    record is [dx_0..dx_{P-1} | dy_0..dy_{P-1} | m_0..m_{P-1}], and point j
 *    sits on grid index k = j for j < (K*K-1)/2 and k = j + 1 after it (the
 *    centre grid index (K*K-1)/2 is skipped);
 *  - centre feature scaling: with a logit z[n,ho,wo,g] given as input,
 *    s = 1 / (1 + exp(-z)) and out = (1 - s) * aggregate + s * x_c, where
 *    x_c is x at the centre grid position (ho*stride - pad + (K/2)*dilation,
 *    wo*stride - pad + (K/2)*dilation) of channel g*Cg + c, zero outside the
 *    image (for stride 1 and pad = dilation*(K-1)/2 that is the output pixel
 *    itself).
 * center_logit: [N,Hout,Wout,G] (read only when center_scale != 0).
 * ------------------------------------------------------------------------ */
int oracle_dcnv4_forward_variants(const double *x, const double *om, const double *center_logit, double *out,
                                  int N, int H, int W, int C, int G, int K,
                                  int stride, int pad, int dilation, float offset_scale,
                                  int softmax, int remove_center, int center_scale)
{
    if (N < 0 || H <= 0 || W <= 0 || C <= 0 || G <= 0 || K <= 0 || K > 16 || C % G) return -1;
    if (remove_center && (K % 2 == 0 || K < 3)) return -1;
    if (center_scale && !center_logit) return -1;
    const int Hout = oracle_output_size(H, K, stride, pad, dilation);
    const int Wout = oracle_output_size(W, K, stride, pad, dilation);
    if (Hout <= 0 || Wout <= 0) return -1;
    const int Cg = C / G, KK = K * K;
    const int centre = (KK - 1) / 2;
    const int P = remove_center ? KK - 1 : KK;
    double mk[256];
    for (int n = 0; n < N; ++n)
        for (int ho = 0; ho < Hout; ++ho)
            for (int wo = 0; wo < Wout; ++wo)
                for (int g = 0; g < G; ++g) {
                    const size_t unit = (((size_t)n * Hout + ho) * Wout + wo) * G + g;
                    const double *r = om + unit * (size_t)(3 * P);
                    double *o = out + (((size_t)n * Hout + ho) * Wout + wo) * (size_t)C + (size_t)g * Cg;
                    /* the aggregation weights, optionally through a softmax over the unit's points */
                    if (softmax) {
                        double mx = r[2 * P];
                        for (int j = 1; j < P; ++j)
                            if (r[2 * P + j] > mx) mx = r[2 * P + j];
                        double sum = 0.0;
                        for (int j = 0; j < P; ++j) sum += exp(r[2 * P + j] - mx);
                        for (int j = 0; j < P; ++j) mk[j] = exp(r[2 * P + j] - mx) / sum;
                    } else {
                        for (int j = 0; j < P; ++j) mk[j] = r[2 * P + j];
                    }
                    for (int c = 0; c < Cg; ++c) o[c] = 0.0;
                    for (int j = 0; j < P; ++j) {
                        const int k = (remove_center && j >= centre) ? j + 1 : j;
                        const int ky = k / K, kx = k % K;
                        const int p0y = ho * stride - pad + ky * dilation;
                        const int p0x = wo * stride - pad + kx * dilation;
                        const double dx = scaled_offset(offset_scale, r[j]);
                        const double dy = scaled_offset(offset_scale, r[P + j]);
                        if (!isfinite(dx) || !isfinite(dy)) continue;
                        const double fy0 = floor(dy), fx0 = floor(dx);
                        const double ly = dy - fy0, lx = dx - fx0;
                        const double y0 = (double)p0y + fy0, x0 = (double)p0x + fx0;
                        for (int a = 0; a <= 1; ++a)
                            for (int b = 0; b <= 1; ++b) {
                                const double yy = y0 + a, xx = x0 + b;
                                if (!(yy >= 0.0 && yy <= (double)(H - 1) && xx >= 0.0 && xx <= (double)(W - 1)))
                                    continue;
                                const double w = mk[j] * (a ? ly : 1.0 - ly) * (b ? lx : 1.0 - lx);
                                const double *px = x + ((((size_t)n * H + (size_t)yy) * W + (size_t)xx) * C) + (size_t)g * Cg;
                                for (int c = 0; c < Cg; ++c) o[c] += w * px[c];
                            }
                    }
                    if (center_scale) {
                        const double sg = 1.0 / (1.0 + exp(-center_logit[unit]));
                        const int cy = ho * stride - pad + (K / 2) * dilation;
                        const int cx = wo * stride - pad + (K / 2) * dilation;
                        const int inside = cy >= 0 && cy < H && cx >= 0 && cx < W;
                        const double *px = x + ((((size_t)n * H + (size_t)(inside ? cy : 0)) * W +
                                                 (size_t)(inside ? cx : 0)) * C) + (size_t)g * Cg;
                        for (int c = 0; c < Cg; ++c) {
                            const double xc = inside ? px[c] : 0.0;
                            o[c] = (1.0 - sg) * o[c] + sg * xc;
                        }
                    }
                }
    return 0;
}

/* ------------------------------------------------------------------------
 * The offset/mask predictor's last step. "不只是卷积的平替" (jsqmd.com),
 * section 2, U-Net block listing: a depthwise 3x3 convolution followed by a
 * 1x1 convolution to 3*groups*9 channels predicts the parameters; the first
 * 2*groups*9 channels are the offsets and the rest the masks, and section 1's
 * listing reads them as offset.reshape(N, G, 2, K*K, ...) and
 * mask.reshape(N, G, K*K, ...). This function is that 1x1 convolution on
 * channels-last input followed by the repacking into this library's
 * offset_mask record:
 *   params[m, o] = bias[o] + sum_c W[o, c] * y[m, c]      (o < 3*G*P)
 *   o = g*2P + comp*P + j  (o < 2GP)  ->  record[m, g, comp*P + j]
 *   o = 2GP + g*P + j                 ->  record[m, g, 2P + j]
 * y: [M, C] (M pixels), W: [3GP, C], bias: [3GP] (NULL: none),
 * record: [M, G, 3P]. P = points per group (K*K, or K*K - 1 without the
 * centre).
 * ------------------------------------------------------------------------ */
int oracle_dcnv4_predictor(const double *y, const double *w, const double *bias, double *record,
                           int M, int C, int G, int P)
{
    if (M < 0 || C <= 0 || G <= 0 || P <= 0) return -1;
    const int NO = 3 * G * P;
    for (int m = 0; m < M; ++m)
        for (int o = 0; o < NO; ++o) {
            double acc = bias ? bias[o] : 0.0;
            for (int c = 0; c < C; ++c) acc += w[(size_t)o * C + c] * y[(size_t)m * C + c];
            int g, slot;
            if (o < 2 * G * P) {
                g = o / (2 * P);
                slot = o % (2 * P);          /* comp * P + j */
            } else {
                g = (o - 2 * G * P) / P;
                slot = 2 * P + (o - 2 * G * P) % P;
            }
            record[((size_t)m * G + g) * (size_t)(3 * P) + slot] = acc;
        }
    return 0;
}

/* ------------------------------------------------------------------------
 * Backward of the forward above (the training direction; the pages use the
 * operator for training, e.g. the Stable Diffusion fine-tuning of the
 * jsqmd.com page, section 4). For a loss L with dL/dout = grad_out:
 *   dL/dx[n,y,x,gc]  = sum over every (ho, wo, k, corner) that reads (y, x) of
 *                      m_k * W_corner * grad_out[n,ho,wo,gc]
 *   dL/dm_k          = sum_c grad_out[c] * sample_k[c],  sample_k = sum_corners W * x
 *   dL/d r[k]        = m_k * s * sum_c grad_out[c] * sum_corners dW/dfx * x   (x-offset)
 *   dL/d r[K*K + k]  = m_k * s * sum_c grad_out[c] * sum_corners dW/dfy * x   (y-offset)
 * with W_ab = (a ? fy : 1-fy) (b ? fx : 1-fx), dW/dfy = (a ? 1 : -1)(b ? fx : 1-fx),
 * dW/dfx = (a ? fy : 1-fy)(b ? 1 : -1), s = offset_scale (d = s*r, and
 * fy = d - floor(d) moves one for one with d between integers). Corners
 * outside the image take no part; a sample with a non-finite offset is
 * outside and gets zero gradients. At an integer position the corner set of
 * floor(d) is used, i.e. the derivative from above.
 * grad_x: [N,H,W,C] (overwritten), grad_om: [N,Hout,Wout,G,3*K*K] (overwritten).
 * ------------------------------------------------------------------------ */
int oracle_dcnv4_backward(const double *x, const double *om, const double *grad_out,
                          double *grad_x, double *grad_om,
                          int N, int H, int W, int C, int G, int K,
                          int stride, int pad, int dilation, float offset_scale)
{
    if (N < 0 || H <= 0 || W <= 0 || C <= 0 || G <= 0 || K <= 0 || C % G) return -1;
    const int Hout = oracle_output_size(H, K, stride, pad, dilation);
    const int Wout = oracle_output_size(W, K, stride, pad, dilation);
    if (Hout <= 0 || Wout <= 0) return -1;
    const int Cg = C / G, KK = K * K;
    for (size_t i = 0; i < (size_t)N * H * W * C; ++i) grad_x[i] = 0.0;
    for (int n = 0; n < N; ++n)
        for (int ho = 0; ho < Hout; ++ho)
            for (int wo = 0; wo < Wout; ++wo)
                for (int g = 0; g < G; ++g) {
                    const size_t unit = (((size_t)n * Hout + ho) * Wout + wo) * G + g;
                    const double *r = om + unit * (size_t)(3 * KK);
                    double *gr = grad_om + unit * (size_t)(3 * KK);
                    const double *go = grad_out + (((size_t)n * Hout + ho) * Wout + wo) * (size_t)C + (size_t)g * Cg;
                    for (int k = 0; k < KK; ++k) {
                        const int ky = k / K, kx = k % K;
                        const int p0y = ho * stride - pad + ky * dilation;
                        const int p0x = wo * stride - pad + kx * dilation;
                        const double dx = scaled_offset(offset_scale, r[k]);
                        const double dy = scaled_offset(offset_scale, r[KK + k]);
                        const double m = r[2 * KK + k];
                        double g_m = 0.0, g_fx = 0.0, g_fy = 0.0;
                        if (isfinite(dx) && isfinite(dy)) {
                            const double fy0 = floor(dy), fx0 = floor(dx);
                            const double ly = dy - fy0, lx = dx - fx0;
                            const double y0 = (double)p0y + fy0, x0 = (double)p0x + fx0;
                            for (int a = 0; a <= 1; ++a)
                                for (int b = 0; b <= 1; ++b) {
                                    const double yy = y0 + a, xx = x0 + b;
                                    if (!(yy >= 0.0 && yy <= (double)(H - 1) && xx >= 0.0 && xx <= (double)(W - 1)))
                                        continue;
                                    const double wy = a ? ly : 1.0 - ly, wx = b ? lx : 1.0 - lx;
                                    const double dwy = a ? 1.0 : -1.0, dwx = b ? 1.0 : -1.0;
                                    const size_t pix = (((size_t)n * H + (size_t)yy) * W + (size_t)xx) * C + (size_t)g * Cg;
                                    for (int c = 0; c < Cg; ++c) {
                                        const double xv = x[pix + c];
                                        g_m += go[c] * wy * wx * xv;
                                        g_fy += go[c] * dwy * wx * xv;
                                        g_fx += go[c] * wy * dwx * xv;
                                        grad_x[pix + c] += m * wy * wx * go[c];
                                    }
                                }
                        }
                        gr[k] = m * (double)offset_scale * g_fx;
                        gr[KK + k] = m * (double)offset_scale * g_fy;
                        gr[2 * KK + k] = g_m;
                    }
                }
    return 0;
}

/* ------------------------------------------------------------------------
 * Backward of oracle_dcnv4_forward_variants (same readings). With
 * m' the (optionally softmax-normalised) masks, s = sigmoid(z) the centre
 * gate (s = 0 without centre scaling) and g = dL/dout:
 *   the aggregation sees g' = (1 - s) g, so grad_x, the offset gradients and
 *   dL/dm'_j = (1 - s) u_j with u_j = sum_c g[c] S_j[c] are those of the plain
 *   backward with masks m' and upstream g';
 *   softmax: dL/dm_j = m'_j (dL/dm'_j - sum_i m'_i dL/dm'_i);
 *   centre scaling: grad_x[centre] += s g and
 *   dL/dz = s (1 - s) (sum_c g[c] x_c[c] - sum_j m'_j u_j).
 * grad_z: [N,Hout,Wout,G] (written only with center_scale).
 * ------------------------------------------------------------------------ */
int oracle_dcnv4_backward_variants(const double *x, const double *om, const double *center_logit,
                                   const double *grad_out, double *grad_x, double *grad_om, double *grad_z,
                                   int N, int H, int W, int C, int G, int K,
                                   int stride, int pad, int dilation, float offset_scale,
                                   int softmax, int remove_center, int center_scale)
{
    if (N < 0 || H <= 0 || W <= 0 || C <= 0 || G <= 0 || K <= 0 || K > 16 || C % G) return -1;
    if (remove_center && (K % 2 == 0 || K < 3)) return -1;
    if (center_scale && (!center_logit || !grad_z)) return -1;
    const int Hout = oracle_output_size(H, K, stride, pad, dilation);
    const int Wout = oracle_output_size(W, K, stride, pad, dilation);
    if (Hout <= 0 || Wout <= 0) return -1;
    const int Cg = C / G, KK = K * K;
    const int centre = (KK - 1) / 2;
    const int P = remove_center ? KK - 1 : KK;
    double mk[256], u[256];
    for (size_t i = 0; i < (size_t)N * H * W * C; ++i) grad_x[i] = 0.0;
    for (int n = 0; n < N; ++n)
        for (int ho = 0; ho < Hout; ++ho)
            for (int wo = 0; wo < Wout; ++wo)
                for (int g = 0; g < G; ++g) {
                    const size_t unit = (((size_t)n * Hout + ho) * Wout + wo) * G + g;
                    const double *r = om + unit * (size_t)(3 * P);
                    double *gr = grad_om + unit * (size_t)(3 * P);
                    const double *go = grad_out + (((size_t)n * Hout + ho) * Wout + wo) * (size_t)C + (size_t)g * Cg;
                    if (softmax) {
                        double mx = r[2 * P];
                        for (int j = 1; j < P; ++j)
                            if (r[2 * P + j] > mx) mx = r[2 * P + j];
                        double sum = 0.0;
                        for (int j = 0; j < P; ++j) sum += exp(r[2 * P + j] - mx);
                        for (int j = 0; j < P; ++j) mk[j] = exp(r[2 * P + j] - mx) / sum;
                    } else {
                        for (int j = 0; j < P; ++j) mk[j] = r[2 * P + j];
                    }
                    const double sg = center_scale ? 1.0 / (1.0 + exp(-center_logit[unit])) : 0.0;
                    for (int j = 0; j < P; ++j) {
                        const int k = (remove_center && j >= centre) ? j + 1 : j;
                        const int ky = k / K, kx = k % K;
                        const int p0y = ho * stride - pad + ky * dilation;
                        const int p0x = wo * stride - pad + kx * dilation;
                        const double dx = scaled_offset(offset_scale, r[j]);
                        const double dy = scaled_offset(offset_scale, r[P + j]);
                        double uj = 0.0, g_fx = 0.0, g_fy = 0.0;
                        if (isfinite(dx) && isfinite(dy)) {
                            const double fy0 = floor(dy), fx0 = floor(dx);
                            const double ly = dy - fy0, lx = dx - fx0;
                            const double y0 = (double)p0y + fy0, x0 = (double)p0x + fx0;
                            for (int a = 0; a <= 1; ++a)
                                for (int b = 0; b <= 1; ++b) {
                                    const double yy = y0 + a, xx = x0 + b;
                                    if (!(yy >= 0.0 && yy <= (double)(H - 1) && xx >= 0.0 && xx <= (double)(W - 1)))
                                        continue;
                                    const double wy = a ? ly : 1.0 - ly, wx = b ? lx : 1.0 - lx;
                                    const double dwy = a ? 1.0 : -1.0, dwx = b ? 1.0 : -1.0;
                                    const size_t pix = (((size_t)n * H + (size_t)yy) * W + (size_t)xx) * C + (size_t)g * Cg;
                                    for (int c = 0; c < Cg; ++c) {
                                        const double xv = x[pix + c];
                                        uj += go[c] * wy * wx * xv;
                                        g_fy += go[c] * dwy * wx * xv;
                                        g_fx += go[c] * wy * dwx * xv;
                                        grad_x[pix + c] += mk[j] * wy * wx * (1.0 - sg) * go[c];
                                    }
                                }
                        }
                        u[j] = uj;
                        gr[j] = mk[j] * (double)offset_scale * (1.0 - sg) * g_fx;
                        gr[P + j] = mk[j] * (double)offset_scale * (1.0 - sg) * g_fy;
                        gr[2 * P + j] = (1.0 - sg) * uj;      /* dL/dm'_j */
                    }
                    if (softmax) {
                        double dot = 0.0;
                        for (int j = 0; j < P; ++j) dot += mk[j] * gr[2 * P + j];
                        for (int j = 0; j < P; ++j) gr[2 * P + j] = mk[j] * (gr[2 * P + j] - dot);
                    }
                    if (center_scale) {
                        const int cy = ho * stride - pad + (K / 2) * dilation;
                        const int cx = wo * stride - pad + (K / 2) * dilation;
                        double gxc = 0.0;
                        if (cy >= 0 && cy < H && cx >= 0 && cx < W) {
                            const size_t pix = (((size_t)n * H + (size_t)cy) * W + (size_t)cx) * C + (size_t)g * Cg;
                            for (int c = 0; c < Cg; ++c) {
                                gxc += go[c] * x[pix + c];
                                grad_x[pix + c] += sg * go[c];
                            }
                        }
                        double mu = 0.0;
                        for (int j = 0; j < P; ++j) mu += mk[j] * u[j];
                        grad_z[unit] = sg * (1.0 - sg) * (gxc - mu);
                    }
                }
    return 0;
}
