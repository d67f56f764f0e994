/*
 * qvae.h -- C ABI of libqvae: the W8A8 CausalConv3d layer of the Qwen-Image /
 * Wan VAE decoder on NVIDIA B200 (sm_100a).
 *
 * The method (ComfyUI-Qwen-VAE-Triton v0.2.0 release note, sd114.wiki):
 *   - opening paragraph: an implicit-GEMM W8A8 kernel for the decoder's
 *     CausalConv3d layers;
 *   - section on the three presets: weights are symmetric INT8 with one scale
 *     per output channel, activations dynamic symmetric INT8, INT8 x INT8
 *     products accumulated in INT32, rescaled in FP32, and the output keeps
 *     the activation's precision; clip ratios 1.0; channels_last; a failing
 *     quantised layer falls back to the native one (here: every call returns
 *     a status and never aborts, the caller decides the fallback);
 *   - the Aggressive preset quantises 26 of 28 layers and leaves 2 in native
 *     precision (here: the `quantized` flag of qvae_layer).
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned.  bf16 tensors are channels_last: [N][T][H][W][C], C fastest.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue work; nothing synchronises the host, and scales stay on the
 *     device.  The library allocates no device memory.
 *   - Return value: QVAE_OK or a qvae_status code.  Argument errors are
 *     detected before anything is launched.  A device-side wait that ran out
 *     of time is reported later by qvae_get_error().
 *   - Layer geometry is fixed: 3x3x3 kernel, stride 1, causal temporal
 *     padding of 2 leading zero frames, spatial padding 1 ("same" size).
 *     The streamed-chunk variant takes two carried frames in place of the
 *     zero frames, the row-band variant halo rows in place of the top and
 *     bottom padding.
 */
#ifndef QVAE_H
#define QVAE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The library is built with hidden visibility; everything declared here is exported. */
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

typedef enum qvae_status {
  QVAE_OK = 0,
  QVAE_ERR_ARG = 1,      /* null pointer, negative size, bad workspace */
  QVAE_ERR_SHAPE = 2,    /* Cin or Cout not a multiple of 32, or sizes out of range */
  QVAE_ERR_ALIGN = 3,    /* a pointer is not 16-byte aligned */
  QVAE_ERR_CUDA = 4,     /* a CUDA call or kernel launch failed */
  QVAE_ERR_TIMEOUT = 5,  /* a device-side pipeline wait ran out of time */
  QVAE_ERR_UNSUPPORTED = 6,
  QVAE_ERR_BOUNDS = 7    /* (debug builds only) a load or store failed its bounds check and was skipped */
} qvae_status;

/* Shape of one CausalConv3d layer; input and output have the same N, T, H, W. */
typedef struct qvae_shape {
  int64_t N, T, H, W;
  int32_t Cin, Cout;
} qvae_shape;

/* Human-readable text of a status code (static storage). */
const char* qvae_status_string(int status);

/* Text of the last CUDA error seen by this library on the calling thread. */
const char* qvae_last_error_message(void);

/* ------------------------------------------------------------- weights -- */

/* Bytes of the packed weight buffer for a layer:
 * 27 taps x ceil(Cin/128) chunks x Cout rows x 128 bytes. */
size_t qvae_packed_weight_bytes(int32_t Cin, int32_t Cout);

/*
 * One-time weight quantisation and repack (release note, three presets:
 * "weights symmetric INT8, one scale per output channel", clip ratio 1.0).
 *   w_bf16     [Cout][Cin][3][3][3] bf16, the PyTorch Conv3d weight layout.
 *   wq_packed  qvae_packed_weight_bytes(Cin, Cout) bytes, written: INT8 codes
 *              in the convolution's consumption order, [tap][chunk][Cout][128]
 *              with tap = (kt*3 + kh)*3 + kw, each 128-byte row holding 128
 *              input channels in the tensor cores' 128-byte swizzle (16-byte
 *              group g at position g ^ (co % 8)), zeros beyond Cin.
 *   w_scale    [Cout] fp32, written: absmax(w[co]) / 127.
 *   wq_plain   optional (NULL to skip): [Cout][27][Cin] codes, tap-major.
 * code = clamp(rint(w / w_scale[co]), -127, 127), IEEE divide, half to even;
 * an all-zero output channel gets scale 0 and zero codes.
 * Needs Cin % 32 == 0 and Cout % 32 == 0.
 */
int qvae_quantize_weights(int32_t Cin, int32_t Cout, const void* w_bf16, int8_t* wq_packed,
                          float* w_scale, int8_t* wq_plain, void* stream);

/* ---------------------------------------------------------- activations -- */

/* Workspace bytes qvae_act_absmax_quant needs (partial maxima); at most 16 KiB. */
size_t qvae_act_workspace_bytes(int64_t numel);

/*
 * Dynamic per-tensor activation quantisation (release note, three presets:
 * "activations dynamic symmetric INT8", clip ratio 1.0).
 *   x_bf16     numel bf16 values (any layout; every element counts).
 *   xq         numel INT8 codes, written in the same order.
 *   x_scale    one fp32 on the device, written: absmax(x) / 127.
 *   workspace  qvae_act_workspace_bytes(numel) bytes of scratch.
 * code = clamp(rint(x / x_scale), -127, 127) with the IEEE divide's result,
 * half to even; an all-zero tensor gets scale 0 and zero codes.  Inputs must
 * be finite.  numel == 0 writes scale 0 and nothing else.
 */
int qvae_act_absmax_quant(const void* x_bf16, int64_t numel, int8_t* xq, float* x_scale,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * qvae_act_absmax_quant without a workspace argument: the same quantisation
 * and outputs, with its scratch (the partial maxima) in a fixed 16 KiB device
 * array inside this library instead of caller memory.  The release note has
 * no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory -- a host runtime that owns every device buffer and
 * hands a layer only its input and output tensors, or a decode loop that may
 * not call cudaMalloc mid-stream (it can block, synchronise the device or fail
 * under memory pressure).  It allocates nothing.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - The array holds 4096 partial maxima, one per block of the absmax pass,
 *     which launches at most 8 blocks per SM: a GPU with more than 512 SMs
 *     would need more and gets QVAE_ERR_UNSUPPORTED with a message.
 *   - Every call on a device shares the one array and leaves the last call's
 *     partial maxima in it; nothing needs clearing because every slot a call
 *     reads is written earlier in the same call.  Calls that overlap on the
 *     GPU (different streams, different host threads) race on the array.
 */
int qvae_act_absmax_quant_noalloc(const void* x_bf16, int64_t numel, int8_t* xq, float* x_scale,
                                  void* stream);

/*
 * The two activation steps apart, for a scale taken over more than the
 * tensor at hand (the row bands of one image, on one GPU or several):
 *   qvae_act_absmax        *amax = max |x| over numel bf16 values, as the
 *                          15-bit magnitude of a bf16 (an unsigned maximum of
 *                          such words is the maximum of the values, so the
 *                          words of several bands or GPUs combine with a
 *                          plain unsigned max, e.g. an all-reduce MAX);
 *                          amax is a device uint32, zeroed by the call.
 *   qvae_act_quant_from_absmax   codes and scale of x for that maximum:
 *                          scale = bf16(amax) / 127, codes as in
 *                          qvae_act_absmax_quant.  With *amax from the whole
 *                          tensor the result equals qvae_act_absmax_quant's.
 * No workspace.  Errors as qvae_act_absmax_quant.
 */
int qvae_act_absmax(const void* x_bf16, int64_t numel, uint32_t* amax, void* stream);
int qvae_act_quant_from_absmax(const void* x_bf16, int64_t numel, const uint32_t* amax, int8_t* xq,
                               float* x_scale, void* stream);

/* ---------------------------------------------------------- convolution -- */

/*
 * The W8A8 causal 3x3x3 convolution (release note: opening paragraph and the
 * three-presets section):
 *   acc[n,t,h,w,co] = sum over kt,kh,kw,ci of
 *                     xq[n, t+kt-2, h+kh-1, w+kw-1, ci] * wq[co, ci, kt, kh, kw]
 *                     (zero outside the tensor), exact in INT32;
 *   out[n,t,h,w,co] = bf16_rne( float(acc) * (x_scale * w_scale[co]) + bias[co] ).
 *   xq         [N][T][H][W][Cin] INT8 codes (from qvae_act_absmax_quant).
 *   x_scale    device fp32 scalar (from qvae_act_absmax_quant).
 *   wq_packed, w_scale   from qvae_quantize_weights.
 *   bias_bf16  [Cout] bf16, or NULL for no bias.
 *   out_bf16   [N][T][H][W][Cout] bf16, written.
 * Needs Cin % 32 == 0, Cout % 32 == 0; sizes with N*T*H*W == 0 do nothing.
 * Ordering: the convolution is launched as a programmatic dependent of the
 * kernel before it on the stream (its set-up overlaps that kernel's tail) and
 * starts loading wq_packed before it waits for that kernel; xq, x_scale,
 * w_scale and bias are read only after the wait.  So wq_packed must not be
 * written by the kernel launched immediately before this call on the same
 * stream.  qvae_quantize_weights keeps this true for its own output (it ends
 * with an empty kernel); copies (cudaMemcpyAsync) and anything with a kernel
 * in between are safe.  The same holds for every convolution entry point
 * below and for qvae_decode_layers.
 */
int qvae_causal_conv3d_w8a8(const qvae_shape* shape, const int8_t* xq, const float* x_scale,
                            const int8_t* wq_packed, const float* w_scale, const void* bias_bf16,
                            void* out_bf16, void* stream);

/* Same convolution, writing the raw INT32 accumulators acc [N][T][H][W][Cout]
 * instead of the bf16 output (for exact checking). */
int qvae_causal_conv3d_w8a8_acc32(const qvae_shape* shape, const int8_t* xq,
                                  const int8_t* wq_packed, int32_t* acc, void* stream);

/*
 * Streamed temporal decode (a video decoded in chunks of frames, as for the
 * Wan VAE the release note names): the same convolution over a chunk of
 * shape->T frames whose input carries, in front of the chunk, the last two
 * input frames of the previous chunk instead of the two causal zero frames:
 *   acc[n,t,h,w,co] = sum over kt,kh,kw,ci of
 *                     xq_ext[n, t+kt, h+kh-1, w+kw-1, ci] * wq[co, ci, kt, kh, kw]
 *   xq_ext     [N][T+2][H][W][Cin] INT8 codes of the extended input, quantised as
 *              one tensor by qvae_act_absmax_quant (so x_scale covers the carried
 *              frames too); frames 0 and 1 are the carried ones.
 *   out_bf16   [N][T][H][W][Cout], the chunk's frames only.
 * With zero carried frames this equals qvae_causal_conv3d_w8a8 on the chunk;
 * with the same codes, chunks that carry their predecessors' last two frames
 * reproduce the whole sequence's accumulators.  Same arguments, layout and
 * errors as qvae_causal_conv3d_w8a8 otherwise.
 */
int qvae_causal_conv3d_w8a8_carry(const qvae_shape* shape, const int8_t* xq_ext, const float* x_scale,
                                  const int8_t* wq_packed, const float* w_scale, const void* bias_bf16,
                                  void* out_bf16, void* stream);

/* The streamed-chunk convolution writing raw INT32 accumulators [N][T][H][W][Cout]. */
int qvae_causal_conv3d_w8a8_carry_acc32(const qvae_shape* shape, const int8_t* xq_ext,
                                        const int8_t* wq_packed, int32_t* acc, void* stream);

/*
 * Row-band decode (tiled decode for memory, which the dsh-qwen-paint plugin
 * README falls back to when a VAE decode runs out of memory; and the split of
 * one image across GPUs): the convolution of output rows [r0, r0 + shape->H),
 * of an image, from an input band holding those rows plus halo_top (0 or 1) rows above
 * and halo_bot (0 or 1) rows below:
 *   xq_band  [N][T][halo_top + H + halo_bot][W][Cin] codes, quantised with the
 *            scale of the whole image (qvae_act_absmax over every band, then
 *            qvae_act_quant_from_absmax per band);
 *   out_bf16 [N][T][H][W][Cout], the band's output rows.
 * A missing halo (0) is the image edge: zero padding.  Output row h reads
 * input rows h + halo_top - 1 .. h + halo_top + 1.  Bands that tile the
 * image, each with the neighbouring rows as halos, give exactly the
 * whole-image convolution.  Errors as qvae_causal_conv3d_w8a8;
 * QVAE_ERR_ARG for a halo outside 0..1.
 */
int qvae_causal_conv3d_w8a8_band(const qvae_shape* shape, int32_t halo_top, int32_t halo_bot,
                                 const int8_t* xq_band, const float* x_scale, const int8_t* wq_packed,
                                 const float* w_scale, const void* bias_bf16, void* out_bf16, void* stream);

/*
 * The W8A8 convolution quantising its bf16 input itself (the quantise step
 * fused into the convolution's producer): x is read once, as bf16, by the
 * convolution, and its codes are made in shared memory -- never written to
 * device memory.  The codes and the scale are those of qvae_act_absmax_quant
 * for the maximum *x_amax:
 *   scale = bf16(*x_amax) / 127,  code = clamp(rint(x / scale), -127, 127),
 * and the output is that of qvae_causal_conv3d_w8a8 on those codes.
 *   x_bf16      [N][T][H][W][Cin] bf16.
 *   x_amax      device uint32: the bf16 magnitude bits of max |x| over the
 *               tensor (qvae_act_absmax writes it), read after the kernel
 *               before this call on the stream has finished.
 *   x_scale_out device fp32, or NULL: receives the activation scale.
 * A layer is then qvae_act_absmax followed by this call: two passes over x
 * instead of the absmax, the quantise pass and the codes' write and read.
 * Same arguments, layout, errors and ordering as qvae_causal_conv3d_w8a8
 * otherwise (x_bf16, like wq_packed, must not be written by the kernel
 * launched immediately before this call).
 */
int qvae_causal_conv3d_w8a8_fused(const qvae_shape* shape, const void* x_bf16, const uint32_t* x_amax,
                                  const int8_t* wq_packed, const float* w_scale, const void* bias_bf16,
                                  void* out_bf16, float* x_scale_out, void* stream);

/* The fused convolution writing raw INT32 accumulators [N][T][H][W][Cout]. */
int qvae_causal_conv3d_w8a8_fused_acc32(const qvae_shape* shape, const void* x_bf16, const uint32_t* x_amax,
                                        const int8_t* wq_packed, int32_t* acc, void* stream);

/* The row-band convolution writing raw INT32 accumulators [N][T][H][W][Cout]. */
int qvae_causal_conv3d_w8a8_band_acc32(const qvae_shape* shape, int32_t halo_top, int32_t halo_bot,
                                       const int8_t* xq_band, const int8_t* wq_packed, int32_t* acc,
                                       void* stream);

/* ------------------------------------------------- native-precision layer -- */

/* Bytes of a native layer's packed bf16 weights:
 * 27 taps x ceil(Cin/64) chunks x Cout rows x 128 bytes. */
size_t qvae_packed_weight_bytes_bf16(int32_t Cin, int32_t Cout);

/*
 * One-time repack of a native-precision layer's weights (no quantisation).
 * The release note's Aggressive preset keeps two decoder convolutions in
 * their original precision (its exclusion rule names
 * decoder.upsamples.14.residual.2 and .residual.6); they run on the same
 * tiled convolution with bf16 operands.
 *   w_bf16    [Cout][Cin][3][3][3] bf16, the PyTorch Conv3d weight layout.
 *   w_packed  qvae_packed_weight_bytes_bf16(Cin, Cout) bytes, written:
 *             [tap][chunk][Cout][64] bf16, tap = (kt*3 + kh)*3 + kw, each
 *             128-byte row holding 64 input channels in the 128-byte swizzle
 *             (16-byte group g at position g ^ (co % 8)), zeros beyond Cin.
 * Needs Cin % 32 == 0 and Cout % 32 == 0.  Ends with an empty kernel, like
 * qvae_quantize_weights (see the ordering note of qvae_causal_conv3d_w8a8).
 */
int qvae_pack_weights_bf16(int32_t Cin, int32_t Cout, const void* w_bf16, void* w_packed, void* stream);

/*
 * The causal 3x3x3 convolution in native precision:
 *   out[n,t,h,w,co] = bf16_rne( acc + bias[co] ),
 *   acc = sum over kt,kh,kw,ci of x[n, t+kt-2, h+kh-1, w+kw-1, ci] * w[co, ci, kt, kh, kw]
 * evaluated on the tensor cores (kind::f16) with bf16 products accumulated
 * in fp32 (zero outside the tensor, as for the W8A8 layer).  The sum is not
 * exact: it differs from the exact value by the fp32 rounding of its
 * accumulation, at most 2^-12 of the sum of |x * w| over the layer's shapes.
 *   x_bf16    [N][T][H][W][Cin] bf16.   w_packed from qvae_pack_weights_bf16.
 *   bias_bf16 [Cout] bf16 or NULL.      out_bf16 [N][T][H][W][Cout] bf16.
 * Errors and ordering as qvae_causal_conv3d_w8a8.
 */
int qvae_causal_conv3d_bf16(const qvae_shape* shape, const void* x_bf16, const void* w_packed,
                            const void* bias_bf16, void* out_bf16, void* stream);

/* The native-precision convolution writing its raw fp32 sums acc [N][T][H][W][Cout]
 * (no bias) instead of the bf16 output. */
int qvae_causal_conv3d_bf16_acc32(const qvae_shape* shape, const void* x_bf16, const void* w_packed,
                                  float* acc, void* stream);

/* ---------------------------------------------------------- layer chain -- */

/*
 * One decoder layer for qvae_decode_layers.  quantized == 0 marks a layer
 * kept in native precision (the release note's Aggressive preset keeps 2 of
 * 28): with wq_packed holding its bf16 weights packed by
 * qvae_pack_weights_bf16 the library runs it with qvae_causal_conv3d_bf16
 * (w_scale unused); with wq_packed == NULL the library skips it and the
 * caller runs it.
 */
typedef struct qvae_layer {
  qvae_shape shape;
  int32_t quantized;
  int32_t reserved;          /* set to 0 */
  const void* x;             /* bf16 [N][T][H][W][Cin] */
  void* out;                 /* bf16 [N][T][H][W][Cout] */
  const void* wq_packed;     /* qvae_quantize_weights (quantized), qvae_pack_weights_bf16 (native) or NULL */
  const float* w_scale;      /* [Cout] (quantized layers) */
  const void* bias;          /* bf16 [Cout] or NULL */
} qvae_layer;

/* Workspace bytes qvae_decode_layers needs for these layers under the
 * current qvae_set_fused_quant setting: the last quantised layer's activation
 * scale (fp32 at byte 0) and three maximum words (bytes 64, 128, 192); with
 * the two-pass path also the activation workspace and the largest quantised
 * input's codes. */
size_t qvae_decode_workspace_bytes(const qvae_layer* layers, int32_t n);

/*
 * In order on one stream, for each quantised layer: the activation absmax +
 * quantise passes into the workspace, then the W8A8 convolution into `out`
 * (with qvae_set_fused_quant(1): the absmax into a workspace word, then the
 * fused convolution, which quantises x itself); for each native layer with
 * packed bf16 weights: the bf16 convolution into `out`; native layers without
 * weights are skipped.
 * All layers are validated before anything is launched.  When a layer's
 * `out` is the next layer's `x` and the next layer is quantised (same N, T,
 * H, W and Cout == next Cin), the convolution also accumulates the maximum
 * bf16 magnitude it writes and the next layer skips its absmax pass: each
 * quantised layer is then one kernel.  Codes, scales and outputs are the
 * same as layer-by-layer qvae_act_absmax_quant + qvae_causal_conv3d_w8a8.
 */
int qvae_decode_layers(const qvae_layer* layers, int32_t n, void* workspace,
                       size_t workspace_bytes, void* stream);

/* -------------------------------------------------------------- control -- */

/*
 * Waits for `stream`, then returns and clears the device error word:
 * QVAE_OK, QVAE_ERR_TIMEOUT (a pipeline wait inside a kernel gave up; the
 * results of that call are invalid), QVAE_ERR_BOUNDS (a library built with
 * -DQVAE_DEBUG_CHECKS found a load or store outside its tensor, ring or
 * accumulator and skipped it; the results are invalid), or QVAE_ERR_CUDA if
 * the wait failed.
 */
int qvae_get_error(void* stream);

/*
 * Time limit of every device-side pipeline wait, in nanoseconds (default
 * 2e9).  A wait past it makes the kernel record QVAE_ERR_TIMEOUT, wait
 * (bounded) for its own copies in flight, free its tensor memory and return.
 */
int qvae_set_wait_limit_ns(uint64_t limit_ns);

/*
 * Launches a kernel whose only wait can never be satisfied, with the given
 * limit: the wait must give up and qvae_get_error() must then report
 * QVAE_ERR_TIMEOUT.  Exercises the timeout path without faulting the GPU.
 */
int qvae_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/*
 * How this library was built: bit 0 set = the kernels' bounds checks are
 * compiled in (libqvae_debug.so, -DQVAE_DEBUG_CHECKS; a failed check makes
 * qvae_get_error() return QVAE_ERR_BOUNDS).  Other bits are zero.
 */
int qvae_build_flags(void);

/*
 * Convolution tiling override for tuning and tests (process-wide, not
 * thread-safe).  A CTA tile is MS sub-tiles of 128 output pixels (16 image
 * rows x 8 columns each, stacked vertically) by NT output channels.
 *   MS    1..4;  NT  a multiple of 32 dividing Cout, <= 256;  MS * NT <= 512
 *   SA/SB activation / weight pipeline stages (<= 12)
 *   mode  1 = one CTA per MMA, 2 = CTA pairs (cta_group::2, M = 256 per MMA)
 *   G     taps per weight stage: 1, or 3 (one kernel row; MS <= 2)
 * Zero = automatic (a cost model over the shape).  A forced value that
 * cannot be used for a shape makes the convolution return an error.
 */
int qvae_set_conv_tiling(int32_t MS, int32_t NT, int32_t SA, int32_t SB, int32_t mode, int32_t G);

/*
 * Cap on the number of convolution CTAs (process-wide, tests and tuning):
 * 0 = the default, one CTA (or CTA pair) per SM up to the number of tiles.
 * A small cap makes each CTA walk several tiles of a small problem.
 */
int qvae_set_conv_cta_limit(int32_t max_ctas);

/*
 * How qvae_decode_layers runs quantised layers (process-wide, tuning and
 * tests): 0 (default) the quantise pass writes codes that the convolution
 * reads; 1 the fused convolution quantises in its producer.  Both give the
 * same codes, scales and outputs; the default is the one that measured
 * faster on B200.  Query qvae_decode_workspace_bytes after changing it.
 */
int qvae_set_fused_quant(int32_t on);

/* The tiling the next convolution of this shape would use: out[0..7] = MS,
 * NT, SA, SB, accumulator buffers (1 or 2), CTAs of work, mode (1 or 2), G.
 * variant: 0 the W8A8 convolution of INT8 codes, 1 the fused W8A8
 * convolution (bf16 input quantised in the kernel), 2 the native-precision
 * convolution. */
int qvae_get_conv_tiling(const qvae_shape* shape, int32_t variant, int32_t* out8);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif

#ifdef __cplusplus
}
#endif

#endif /* QVAE_H */
