/*
 * dcnv4.h -- C ABI of libdcnv4.so, the B200 (sm_100a) DCNv4 forward spatial
 * aggregation and its backward.
 *
 * The operation (sources by page title and section):
 *   "不只是卷积的平替：我把DCNv4塞进Stable Diffusion的U-Net里" (jsqmd.com),
 *   section 1: DCNv4 drops the softmax over the aggregation weights, so the
 *   per-point modulation scalars are used as they are (any sign, any size);
 *   its simplified forward listing adds learned offsets to a regular K x K
 *   grid, samples the input bilinearly at the moved points and sums the
 *   samples weighted by the masks, separately for each channel group.
 *   "掌握DCNv4技术：3倍速度提升与80%加速效果的实战指南" (pwwt.cn), tuning
 *   section: offset_scale multiplies the offsets; group sets the number of
 *   channel groups.
 *
 * For output pixel (n, ho, wo), group g (channels [g*Cg, (g+1)*Cg), Cg = C/G)
 * and grid point k = ky*K + kx (row-major), with r = offset_mask[n,ho,wo,g,:]:
 *   p0y = ho*stride - pad + ky*dilation,  p0x = wo*stride - pad + kx*dilation
 *   dx  = fl32(offset_scale * r[k]),      dy  = fl32(offset_scale * r[K*K + k])
 *   m   = r[2*K*K + k]                    (raw modulation scalar, no softmax)
 *   out[n,ho,wo,g*Cg + c] = sum_k m * bilinear(x[n,:,:,g*Cg + c], p0y + dy, p0x + dx)
 * where bilinear() reads zero outside the image, corner by corner: corners
 * (y0+a, x0+b), y0 = p0y + floor(dy), x0 = p0x + floor(dx), a,b in {0,1},
 * weighted (a ? fy : 1-fy) * (b ? fx : 1-fx), fy = dy - floor(dy),
 * fx = dx - floor(dx). Corners inside the image always take part (also with
 * weight 0); a non-finite offset puts the whole sample outside. The corner
 * weight m * (1-fy or fy) * (1-fx or fx) is computed in fp32. For fp32 and
 * bf16 storage it multiplies x in fp32; for fp16 storage it is rounded once to
 * fp16 and the fp16 x fp16 product, exact in fp32, is accumulated by a
 * mixed-precision FMA. Sums are fp32; the result is rounded once
 * (round-to-nearest-even) to the storage type.
 *
 * Layouts (all contiguous, row-major, caller-owned DEVICE memory unless
 * stated otherwise):
 *   x           [N, H, W, C]                  channels-last
 *   offset_mask [N, Hout, Wout, G, 3*K*K]     per group: K*K x-offsets (along
 *                                             the width), K*K y-offsets, K*K masks
 *   out         [N, Hout, Wout, C]
 * with Hout = (H + 2*pad - dilation*(K-1) - 1)/stride + 1 (the same for W).
 * x, offset_mask and out share one storage type (dtype).
 *
 * Conventions:
 *   - Every call is thread-safe; the library keeps no pointer to caller
 *     memory after return and allocates no device memory (the probes below
 *     excepted). It caches, in host memory and per geometry, storage type
 *     and SM count, the forward's choice of kernel plan (and, for the
 *     host-memory entry points, three streams per device and whether a
 *     geometry's bands of output rows take the whole image's plan); each
 *     cache is guarded by its own lock.
 *   - Compute calls are asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and never synchronise. Arguments are checked on
 *     the host before anything is launched; on a non-zero return nothing was
 *     launched (except DCNV4_ERR_LAUNCH, reported when the launch itself
 *     failed).
 *   - Buffer sizes cannot be checked through raw pointers: the caller
 *     guarantees each buffer holds the element count its layout implies.
 *   - NaN / Inf inside x or the masks are data, not errors.
 */
#ifndef DCNV4_H
#define DCNV4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DCNV4_ABI_VERSION 1

/* symbols of the shared library (it is built with hidden default visibility) */
#if defined(__GNUC__)
#define DCNV4_API __attribute__((visibility("default")))
#else
#define DCNV4_API
#endif

/* Storage type of x, offset_mask and out. Sums are fp32 in every case; the
 * corner weights are fp32 for DCNV4_F32 and DCNV4_BF16 and are rounded once to
 * fp16 for DCNV4_F16 (fp16 x fp16 products, exact in fp32, accumulated in
 * fp32), as stated with the formula above. */
typedef enum {
    DCNV4_F32 = 0,
    DCNV4_F16 = 1,
    DCNV4_BF16 = 2
} dcnv4_dtype_t;

typedef enum {
    DCNV4_OK = 0,
    DCNV4_ERR_NULL = 1,      /* a required pointer is NULL (N > 0)                      */
    DCNV4_ERR_SHAPE = 2,     /* N < 0; H, W, C, G, K, stride or dilation <= 0; pad < 0;  */
                             /* Hout or Wout <= 0; K > DCNV4_MAX_K; a spatial extent or  */
                             /* grid coordinate beyond DCNV4_MAX_EXTENT                  */
    DCNV4_ERR_GROUPS = 3,    /* C is not a multiple of G                                */
    DCNV4_ERR_DTYPE = 4,     /* dtype is not a dcnv4_dtype_t value                      */
    DCNV4_ERR_ALIGN = 5,     /* a pointer is not aligned to its element size            */
    DCNV4_ERR_ALIAS = 6,     /* an output buffer overlaps an input buffer               */
    DCNV4_ERR_SCALE = 7,     /* offset_scale is NaN or infinite                         */
    DCNV4_ERR_TOO_LARGE = 8, /* an element count reaches 2^31                           */
    DCNV4_ERR_LAUNCH = 9,    /* the kernel launch failed (CUDA error after launch)      */
    DCNV4_ERR_CUDA = 10,     /* a CUDA runtime call other than a launch failed          */
    DCNV4_ERR_STAGING = 11,  /* dcnv4_forward_host_noalloc: one image does not fit its  */
                             /* half of the library's static staging area               */
    DCNV4_ERR_FLAGS = 12     /* dcnv4_forward_ex: a flag bit that is not defined        */
} dcnv4_status_t;

/* Variant switches of dcnv4_forward_ex / dcnv4_validate_ex (bitwise or).
 * Sources: "掌握DCNv4技术" (pwwt.cn), section on advanced tuning and extension
 * (DCNv4 also offers centre feature scaling, a sigmoid that weighs the centre
 * feature, and removal of the centre point); "不只是卷积的平替" (jsqmd.com),
 * section 1 (DCNv3 normalised the aggregation weights with a softmax, which
 * DCNv4 removed). The pages give no formulas; the readings are:
 *   DCNV4_FLAG_SOFTMAX: per (n, ho, wo, g) the masks are replaced by
 *     m'_j = exp(m_j - max) / sum_i exp(m_i - max) over the unit's points
 *     (fp32, expf), then aggregated as usual;
 *   DCNV4_FLAG_REMOVE_CENTER: K odd and >= 3; each unit has P = K*K - 1
 *     points, offset_mask is [N,Hout,Wout,G,3*P] with per group P x-offsets,
 *     P y-offsets, P masks, and point j sits on grid index j before the
 *     centre (K*K-1)/2 and j + 1 after it;
 *   DCNV4_FLAG_CENTER_SCALE: with s = 1/(1 + exp(-center_logit[n,ho,wo,g])),
 *     out = (1 - s) * aggregate + s * x_c, x_c being x at the centre grid
 *     position (ho*stride - pad + (K/2)*dilation, wo*stride - pad +
 *     (K/2)*dilation), channels of group g, zero outside the image. */
#define DCNV4_FLAG_SOFTMAX 1u
#define DCNV4_FLAG_REMOVE_CENTER 2u
#define DCNV4_FLAG_CENTER_SCALE 4u

#define DCNV4_MAX_K 16
#define DCNV4_MAX_EXTENT (1 << 22)

/* Output extent, convolution style (the formula above).
 * Writes *Hout, *Wout (either may be NULL) and returns DCNV4_OK, or
 * DCNV4_ERR_SHAPE when an argument is out of range or an extent would be <= 0
 * (outputs are then left untouched). Host only; no CUDA call. */
DCNV4_API int dcnv4_output_shape(int H, int W, int K, int stride, int pad, int dilation,
                       int *Hout, int *Wout);

/* Checks the arguments of dcnv4_forward without launching anything.
 * Pointers are only compared (NULL, alignment to the element size, overlap of
 * out with x or offset_mask over the byte ranges their shapes imply); they
 * are never dereferenced. N == 0 is valid (pointers may then be NULL).
 * Returns DCNV4_OK or the first failing dcnv4_status_t. Host only. */
DCNV4_API int dcnv4_validate(const void *x, const void *offset_mask, const void *out,
                   int N, int H, int W, int C, int G, int K,
                   int stride, int pad, int dilation, float offset_scale, int dtype);

/* The forward aggregation (the formula above) for the whole batch.
 * x, offset_mask: read only; out: fully overwritten. All three are device
 * pointers in the layouts above. Runs dcnv4_validate first and returns its
 * code without launching when it fails. On success one kernel is launched
 * on `stream` (none when N == 0) and DCNV4_OK is returned; the result is
 * ready when the stream reaches that point. The launch uses programmatic
 * stream serialisation: its CTAs may start while the previous kernel on the
 * stream finishes, and wait for that kernel to complete before they read or
 * write global memory, so stream order holds as for any launch. */
DCNV4_API int dcnv4_forward(const void *x, const void *offset_mask, void *out,
                  int N, int H, int W, int C, int G, int K,
                  int stride, int pad, int dilation, float offset_scale, int dtype,
                  void *stream);

/* dcnv4_validate with the variant flags above: additionally DCNV4_ERR_FLAGS
 * for an unknown bit, DCNV4_ERR_SHAPE for DCNV4_FLAG_REMOVE_CENTER with an
 * even K or K < 3, and, with DCNV4_FLAG_CENTER_SCALE, center_logit (type
 * dtype, [N,Hout,Wout,G]) non-NULL, aligned and not overlapping out.
 * center_logit is ignored (may be NULL) without DCNV4_FLAG_CENTER_SCALE.
 * offset_mask's size follows the flags (3*(K*K-1) per group without the
 * centre). Host only. */
DCNV4_API int dcnv4_validate_ex(const void *x, const void *offset_mask, const void *center_logit,
                      const void *out, int N, int H, int W, int C, int G, int K,
                      int stride, int pad, int dilation, float offset_scale, int dtype,
                      unsigned int flags);

/* dcnv4_forward with the variant flags above (flags == 0 is dcnv4_forward).
 * center_logit: device, read only, [N,Hout,Wout,G] of type dtype, used only
 * with DCNV4_FLAG_CENTER_SCALE. Same launch, ownership and error behaviour
 * as dcnv4_forward, after dcnv4_validate_ex. */
DCNV4_API int dcnv4_forward_ex(const void *x, const void *offset_mask, const void *center_logit, void *out,
                     int N, int H, int W, int C, int G, int K,
                     int stride, int pad, int dilation, float offset_scale, int dtype,
                     unsigned int flags, void *stream);

/* The backward of dcnv4_forward, for training with the operator ("不只是卷积的
 * 平替：我把DCNv4塞进Stable Diffusion的U-Net里", jsqmd.com: section 1 defines the
 * forward, section 4 fine-tunes through it). For a loss L with
 * dL/dout = grad_out it writes
 *   grad_x[n,y,x,c]   = sum over the in-bounds corners (y, x) of every point
 *                       that reads them of m_k * W_corner * grad_out[...,c],
 *   grad_offset_mask  = per (n, ho, wo, g) record, the same layout as
 *                       offset_mask: [m_k*s*dL/dfx_k (K*K) | m_k*s*dL/dfy_k
 *                       (K*K) | dL/dm_k (K*K)], dL/dm_k being the sum over
 *                       the group's channels of grad_out times the bilinear
 *                       sample, and dL/dfx_k, dL/dfy_k the derivatives of that
 *                       sum with respect to the fractional parts of the
 *                       sample position (s = offset_scale). At an integer
 *                       position the cell of floor(s*r) is used (the
 *                       derivative from above); a point whose offset is not
 *                       finite or that has no corner inside gets zero offset
 *                       and mask gradients and adds nothing to grad_x.
 * x: device, T [N,H,W,C]; offset_mask: device, T [N,Hout,Wout,G,3*K*K];
 * grad_out: device, T [N,Hout,Wout,C] (read only, may overlap x or
 * offset_mask); grad_x: device, fp32 [N,H,W,C], fully overwritten (cleared on
 * `stream` first); grad_offset_mask: device, fp32 [N,Hout,Wout,G,3*K*K],
 * fully overwritten. All buffers are caller-owned; nothing is allocated or
 * kept. Arithmetic is fp32. grad_x sums its contributions with fp32
 * reductions whose order is not fixed, so it can differ in the last bits
 * from run to run; grad_offset_mask is deterministic.
 * Checks as dcnv4_validate (with grad_out in place of out), plus: grad_x and
 * grad_offset_mask non-NULL and 4-byte aligned, overlapping neither each
 * other nor any input (DCNV4_ERR_ALIAS). On success a clear and one kernel
 * are queued on `stream` (nothing when N == 0) and DCNV4_OK is returned. */
DCNV4_API int dcnv4_backward(const void *x, const void *offset_mask, const void *grad_out,
                   float *grad_x, float *grad_offset_mask,
                   int N, int H, int W, int C, int G, int K,
                   int stride, int pad, int dilation, float offset_scale, int dtype,
                   void *stream);

/* The offset/mask predictor's last step: the 1x1 projection of the block's
 * parameter network, packed into offset_mask records. "不只是卷积的平替"
 * (jsqmd.com), section 2: a depthwise 3x3 convolution then a 1x1 convolution
 * to 3*groups*9 channels predict the parameters, the first 2*groups*9 being
 * the offsets and the rest the masks; section 1's listing reads them as
 * offset.reshape(N, G, 2, K*K, ...) and mask.reshape(N, G, K*K, ...). With
 * P = K*K points per group (K*K - 1 with DCNV4_FLAG_REMOVE_CENTER, the only
 * flag taken here) and NO = 3*G*P:
 *   params[m, o] = bias[o] + sum_c weight[o, c] * y[m, c]
 *   offset_mask[m, g, comp*P + j] = params[m, g*2P + comp*P + j]  (comp 0: x, 1: y)
 *   offset_mask[m, g, 2P + j]     = params[m, 2GP + g*P + j]
 * y: device, dtype, [M, C] (M pixels, e.g. N*Hout*Wout, channels-last: the
 * depthwise convolution's output); weight: device, dtype, [NO, C];
 * bias: device fp32 [NO] or NULL; offset_mask: device, dtype, [M, G, 3P],
 * fully overwritten. fp32 sums, one rounding to dtype. fp16/bf16 with C a
 * multiple of 64, NO <= 256 and 16-byte aligned pointers run on the tensor
 * cores (tcgen05.mma, fp32 accumulators in tensor memory); other shapes and
 * fp32 run a CUDA-core kernel. Errors: DCNV4_ERR_SHAPE (M < 0, C, G or K out
 * of range, no centre to remove), DCNV4_ERR_FLAGS, DCNV4_ERR_DTYPE,
 * DCNV4_ERR_TOO_LARGE (an element count >= 2^31), DCNV4_ERR_NULL,
 * DCNV4_ERR_ALIGN, DCNV4_ERR_ALIAS (offset_mask overlaps an input).
 * Asynchronous on `stream`; nothing is launched when M == 0. */
DCNV4_API int dcnv4_predictor(const void *y, const void *weight, const float *bias, void *offset_mask,
                    int M, int C, int G, int K, unsigned int flags, int dtype, void *stream);

/* dcnv4_backward for the variant flags of dcnv4_forward_ex (flags == 0 is
 * dcnv4_backward). With m' the masks the aggregation used (softmax-normalised
 * with DCNV4_FLAG_SOFTMAX) and s = sigmoid(center_logit) (0 without centre
 * scaling), the aggregation's gradients are those of dcnv4_backward with
 * masks m' and upstream (1 - s) * grad_out; the mask block of
 * grad_offset_mask holds dL/dm, i.e. with the softmax's Jacobian applied:
 * m'_j (dL/dm'_j - sum_i m'_i dL/dm'_i). With DCNV4_FLAG_CENTER_SCALE,
 * grad_x additionally receives s * grad_out at the centre grid position
 * (when inside the image) and grad_center_logit[n,ho,wo,g] (device fp32
 * [N,Hout,Wout,G], fully overwritten) = s (1 - s) (sum_c grad_out * x_c -
 * sum_j m'_j u_j), u_j = sum_c grad_out * S_j. Without the centre point the
 * records have 3*(K*K-1) entries per group, as in dcnv4_forward_ex.
 * center_logit and grad_center_logit are needed (non-NULL, aligned, not
 * overlapping any other buffer) only with DCNV4_FLAG_CENTER_SCALE. Other
 * checks, conventions and launch behaviour as dcnv4_backward. */
DCNV4_API int dcnv4_backward_ex(const void *x, const void *offset_mask, const void *center_logit,
                      const void *grad_out, float *grad_x, float *grad_offset_mask,
                      float *grad_center_logit, int N, int H, int W, int C, int G, int K,
                      int stride, int pad, int dilation, float offset_scale, int dtype,
                      unsigned int flags, void *stream);

/* The integer half of the forward, exposed so that it can be compared bit for
 * bit: for every sampling point (n, ho, wo, g, k) it writes the top-left
 * corner (y0, x0) into corner[2*p], corner[2*p+1] and a 4-bit mask of the
 * corners inside the image into valid[p] (bit 0: (y0,x0), bit 1: (y0,x0+1),
 * bit 2: (y0+1,x0), bit 3: (y0+1,x0+1)), p = (((n*Hout+ho)*Wout+wo)*G+g)*K*K+k.
 * A point with no corner inside reports corner = (INT32_MIN, INT32_MIN).
 * corner: device int32 [N,Hout,Wout,G,K*K,2]; valid: device uint8
 * [N,Hout,Wout,G,K*K]. The coordinates are computed by the same device code
 * that the forward kernels use. Same checks as dcnv4_forward with C = G
 * (x is not read; the x and out checks do not apply). */
DCNV4_API int dcnv4_sampling_index(const void *offset_mask, int32_t *corner, uint8_t *valid,
                         int N, int H, int W, int G, int K,
                         int stride, int pad, int dilation, float offset_scale, int dtype,
                         void *stream);

/* The forward of dcnv4_forward, traced: the same plan, kernel code and
 * arithmetic (out receives the same bits as dcnv4_forward writes), and for
 * every sampling point p = (((n*Hout+ho)*Wout+wo)*G+g)*K*K+k the integer
 * corner and validity that the gather actually used, for bit-exact comparison
 * with a reference ("不只是卷积的平替", jsqmd.com, section 1: the sample sits at
 * the regular grid position plus the learned offset):
 *   trace[4p+0], trace[4p+1] = top-left corner (y0, x0), or (INT32_MIN,
 *                              INT32_MIN) when no corner is inside the image;
 *   trace[4p+2]              = validity bits as in dcnv4_sampling_index;
 *   trace[4p+3]              = path: 0 = read from the shared-memory window
 *                              of the ring kernel (validity is then the image
 *                              test that the window's zero fill implements),
 *                              1 = the ring kernel's global-memory pass,
 *                              2 = the global-gather kernel (shapes the ring
 *                              kernel does not take; traced by the index code
 *                              that kernel shares).
 * trace: device int32 [N,Hout,Wout,G,K*K,4], 16-byte aligned, overlapping no
 * other buffer (DCNV4_ERR_NULL / DCNV4_ERR_ALIGN / DCNV4_ERR_ALIAS); other
 * checks as dcnv4_forward, plus DCNV4_ERR_TOO_LARGE when 4*N*Hout*Wout*G*K*K
 * reaches 2^31. A debugging and testing entry point: the tracing kernel is a
 * separate build of the forward kernel with the trace stores compiled in.
 * Asynchronous on `stream`; nothing is launched when N == 0. */
DCNV4_API int dcnv4_forward_trace(const void *x, const void *offset_mask, void *out, int32_t *trace,
                                  int N, int H, int W, int C, int G, int K,
                                  int stride, int pad, int dilation, float offset_scale, int dtype,
                                  void *stream);

/* The forward from and to HOST memory, for callers whose data lives on the
 * host. x_host, offset_mask_host: inputs in host memory (pinned memory lets
 * the copies run asynchronously and overlap; pageable memory works but the
 * copies then block the calling thread); out_host: host memory receiving the
 * result. x_dev, offset_mask_dev, out_dev: caller-owned device buffers of the
 * full sizes of x, offset_mask and out, used as staging (their contents
 * afterwards: the copied inputs and the result). The batch is split into
 * chunks of whole images (about 8 MiB of input copies each, 2 to 8 of them;
 * a batch of fewer images than that is cut into bands of output rows, each
 * band one launch over its rows of the whole image, with the same result bit
 * for bit) and the work is queued on three library-owned non-blocking streams
 * (created once per device on first use and kept until exit), one per role:
 * the host-to-device copies back to back on the first (all of x in one copy
 * ahead of the chunks' offset_mask copies when an image's result is no
 * larger than its offset_mask, else each chunk's x and offset_mask), each
 * chunk's kernel on the second once its inputs have arrived, each chunk's
 * device-to-host copy on the third once its kernel is done; so the two copy
 * directions and the kernels overlap. The call
 * is ordered after the work already queued on `stream`, and `stream` waits for
 * all of it before its next work: synchronise `stream` before reading
 * out_host. Checks: those of dcnv4_forward on the device buffers, plus NULL
 * host pointers (DCNV4_ERR_NULL) and out_host overlapping x_host or
 * offset_mask_host (DCNV4_ERR_ALIAS). A failing CUDA copy, event or stream
 * call returns DCNV4_ERR_CUDA. After any error return that came once copies
 * were queued, `stream` still waits for everything the call queued, so
 * out_host may have been written in part when `stream` reaches that point;
 * synchronise `stream` before reusing or freeing the buffers. The library's
 * streams and cached device addresses belong to the CUDA context current at
 * the first call on each device: the library must not be used after
 * cudaDeviceReset (or any other destruction of that context) in the same
 * process. */
DCNV4_API int dcnv4_forward_host(const void *x_host, const void *offset_mask_host, void *out_host,
                                 void *x_dev, void *offset_mask_dev, void *out_dev,
                                 int N, int H, int W, int C, int G, int K,
                                 int stride, int pad, int dilation, float offset_scale, int dtype,
                                 void *stream);

/* Allocation-free variant of dcnv4_forward_host (the pages have no
 * counterpart: this is a service of this library). Some callers cannot
 * allocate device memory when they call us: a serving process that handed all
 * free GPU memory to its own pool at start-up (a fresh cudaMalloc would fail or
 * fragment that budget), or a latency-critical path where cudaMalloc/cudaFree
 * may synchronise the device and stall other streams. They can use this entry
 * point, which takes only the host buffers: it stages through a fixed device
 * array inside the library, DCNV4_NOALLOC_STAGING_BYTES (32 MiB) per GPU,
 * allocated when the library's device code is loaded on that GPU and kept
 * until the process exits. It never calls cudaMalloc, cudaFree or an
 * allocating library routine.
 *   - The array is split into two halves; the batch is processed in chunks of
 *     whole images, each chunk's x, offset_mask and out (each rounded up to
 *     256 bytes) in one half. A batch whose single image does not fit in one
 *     half (16 MiB) is rejected with DCNV4_ERR_STAGING before anything is
 *     queued.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and keeps it; make that
 *     first call before any stream capture on the device.
 *   - Every call on a device shares the one array and it keeps the last call's
 *     contents; nothing in it needs to start at zero (inputs are copied in
 *     whole, the output is written in whole). Calls whose work overlaps on the
 *     GPU race on the array: queue them on one stream, or order them.
 *   - Chunks alternate between two of the library's streams, one staging
 *     half each (a chunk's copies in, kernel and copy out on one stream).
 *   - Ordering and the other checks are those of dcnv4_forward_host
 *     (the host pointers are checked for NULL, alignment and overlap); the
 *     result is in out_host once `stream` reaches the end of the call's work. After an error return
 *     that came once copies were queued, `stream` still waits for them (see
 *     dcnv4_forward_host). As there, do not use the library after
 *     cudaDeviceReset in the same process: the array's cached address and the
 *     library's streams belong to the context that the first call saw. */
#define DCNV4_NOALLOC_STAGING_BYTES (32u << 20)
DCNV4_API int dcnv4_forward_host_noalloc(const void *x_host, const void *offset_mask_host, void *out_host,
                                         int N, int H, int W, int C, int G, int K,
                                         int stride, int pad, int dilation, float offset_scale, int dtype,
                                         void *stream);

/* Device-side status word of the current device (bit flags below). The
 * shared-memory window kernel waits for its bulk copies with a time limit
 * (1 s); if a wait ever gives up, the CTA sets DCNV4_DEVSTATUS_COPY_TIMEOUT,
 * waits once more (bounded) for copies in flight and leaves its tile
 * unwritten, so a stuck copy shows up here instead of as a hung GPU.
 * Reads the word into *status (synchronous: waits for the device) and, when
 * `clear` is non-zero, resets it to 0. Returns DCNV4_OK, DCNV4_ERR_NULL or
 * DCNV4_ERR_CUDA. */
#define DCNV4_DEVSTATUS_COPY_TIMEOUT 1u
#define DCNV4_DEVSTATUS_SELFTEST_TIMEOUT 2u
DCNV4_API int dcnv4_device_status(unsigned int *status, int clear);

/* Exercises the bounded wait without any fault: one CTA arms an mbarrier for
 * 16 bytes that are never sent, waits `limit_ns` nanoseconds (1 ns .. 2 s),
 * sets DCNV4_DEVSTATUS_SELFTEST_TIMEOUT and returns. Asynchronous on `stream`.
 * Returns DCNV4_OK, DCNV4_ERR_SHAPE (limit out of range) or DCNV4_ERR_LAUNCH. */
DCNV4_API int dcnv4_selftest_wait_timeout(unsigned long long limit_ns, void *stream);

/* Measures this GPU's shared-memory gather rate, the ceiling of the forward
 * kernel's inner loop (each sampling point reads 4 corners x C/G channels from
 * shared memory). The pages have no counterpart; it backs the roofline
 * discussion of the measurements. One CTA per SM, 512 threads, 64 KB of shared
 * memory; every 16-byte load of a quarter warp falls on a different bank
 * position (one 128-byte wavefront per quarter warp and load). pattern 0:
 * independent rows picked at random; pattern 1: the forward's own access
 * pattern (2x2 corners x 2 chunks of 128-byte pixels at random window
 * positions, chunk rotation as in the ring kernel). Writes the bytes moved per
 * SM clock per SM (the slowest CTA's clock64 span). Synchronous: runs on the
 * legacy default stream and waits for the device. Returns DCNV4_OK,
 * DCNV4_ERR_NULL, DCNV4_ERR_SHAPE (unknown pattern), DCNV4_ERR_LAUNCH or
 * DCNV4_ERR_CUDA. */
DCNV4_API int dcnv4_probe_smem_gather(int pattern, double *bytes_per_clock_per_sm);

/* Measures this GPU's rate of fp32 vector reductions into L2, the ceiling of
 * the backward's scatter into grad_x (each sampling point adds m * W * dL/dout
 * to 4 corners x C/G fp32 channels). The pages have no counterpart; it backs
 * the roofline discussion of the backward. One CTA of 512 threads per SM;
 * each warp instruction is a 16-byte `red.global.add.v4.f32` per lane, lanes
 * grouped so that each group covers one segment of `segment_bytes` (32, 64 or
 * 128) contiguous bytes at a random segment of a 32 MB buffer (resident in
 * L2). Writes the payload bytes per SM clock per SM (the slowest CTA's clock64
 * span). Allocates and frees its buffer; synchronous (legacy default stream,
 * waits for the device). Returns DCNV4_OK, DCNV4_ERR_NULL, DCNV4_ERR_SHAPE
 * (segment size not 32, 64 or 128), DCNV4_ERR_LAUNCH or DCNV4_ERR_CUDA. */
DCNV4_API int dcnv4_probe_red_global(int segment_bytes, double *bytes_per_clock_per_sm);

/* Measures this GPU's rate of atomic adds to shared memory, which decides
 * whether a backward could sum grad_x contributions in shared memory before
 * sending them to L2. The pages have no counterpart. One CTA of 512 threads per
 * SM; each thread adds 1 to a word of a 32 KB shared array, every lane of a
 * warp on its own bank; fp32 != 0: `atomicAdd` on fp32 words, else on 32-bit
 * unsigned words. Writes the adds per SM clock per SM (the slowest CTA's
 * clock64 span). Synchronous (legacy default stream, waits for the device).
 * Returns DCNV4_OK, DCNV4_ERR_NULL, DCNV4_ERR_SHAPE (fp32 not 0 or 1),
 * DCNV4_ERR_LAUNCH or DCNV4_ERR_CUDA. */
DCNV4_API int dcnv4_probe_red_shared(int fp32, double *adds_per_clock_per_sm);

/* The forward's plan for a geometry, without launching anything or touching
 * the GPU (the kernel choice and the ring kernel's shape that dcnv4_forward /
 * dcnv4_forward_ex would use with 16-byte-aligned pointers on a GPU of `nsm`
 * SMs, 1..1024). Writes DCNV4_PLAN_FIELDS ints to `fields` (nfields >= that):
 *   [0] kernel: 0 the ring kernel, 1 the global-gather kernel (the other fields 0)
 *   [1] 1: image windows (the whole image plus a one-pixel border), 0: unit windows
 *   [2] halo R of the unit windows   [3] groups per strip      [4] output columns per band
 *   [5] output rows per item         [6] ring rows             [7] items in flight
 *   [8] units (pixel, group) per item  [9] threads per CTA     [10] dynamic shared memory (bytes)
 *   [11] window rows and [12] columns of a unit (image windows: H + 2, W + 2)
 *   [13] window pixels per ring row  [14] bytes per window pixel
 * The planner overrides of the environment (DCNV4_WINDOW, DCNV4_HALO,
 * DCNV4_TILE, DCNV4_GS, DCNV4_NREC, DCNV4_RING) apply as in the forward.
 * Returns DCNV4_OK or the first failing check of dcnv4_validate_ex's sizes
 * and flags, DCNV4_ERR_NULL (fields) or DCNV4_ERR_SHAPE (nfields or nsm). */
#define DCNV4_PLAN_FIELDS 15
DCNV4_API int dcnv4_forward_plan(int N, int H, int W, int C, int G, int K, int stride, int pad, int dilation,
                                 int dtype, unsigned flags, int nsm, int *fields, int nfields);

/* Static description of an error code; never NULL. */
DCNV4_API const char *dcnv4_strerror(int status);

/* DCNV4_ABI_VERSION of the built library. */
DCNV4_API int dcnv4_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DCNV4_H */
