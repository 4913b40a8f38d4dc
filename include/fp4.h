/*
 * fp4.h -- C ABI of the B200 (sm_100a) microscaling FP4 library (libfp4.so).
 *
 * What the operations are (sources, by page and section):
 *  - "FP4 All the Way: Fully Quantized Training of LLMs", Abstract: FP4 (E2M1)
 *    for weights, activations and gradients; NVFP4 = blocks of 16 E2M1 values
 *    sharing an E4M3 scale; round-to-nearest forward, stochastic rounding for
 *    the backward and update passes; block size, scale format and rounding are
 *    the design choices.
 *  - "Bridging the Gap Between Promise and Performance for Microscaling FP4
 *    Quantization", Abstract: MXFP4 (power-of-two scales) and NVFP4;
 *    block-wise Hadamard rotations fused into the weights and computed online
 *    for the activations; FP4 GEMM kernels on B200.
 *  - "Oscillation-Reduced MXFP4 Training for Vision Transformers", Abstract:
 *    MX fine-grained per-group scaling, supported by Blackwell.
 *
 * Encodings (the pages fix none; OCP MX v1.0 conventions are used):
 *  - E2M1 code: bit 3 sign, magnitudes 0,0.5,1,1.5,2,3,4,6 for codes 0..7.
 *    Two codes per byte: element 2j in the low nibble, 2j+1 in the high one.
 *  - MXFP4: 32-element blocks, E8M0 scale byte b (2^(b-127)),
 *    E = clamp(floor(log2 amax_b) - 2, -127, 127); byte 0 for all-zero blocks.
 *  - NVFP4: 16-element blocks, E4M3 scale sb = RNE_sat((amax_b/6)/s_t) under a
 *    per-tensor fp32 scale s_t = amax/(6*448) (1.0 for an all-zero tensor).
 *  - RTN = round to nearest, ties to even code, saturating at +-6, sign kept.
 *    SR = Philox4x32-10 (Salmon et al., SC'11), key = seed, counter =
 *    (idx>>2 as 64-bit, 0, 0), the element with row-major input index idx
 *    takes output word idx&3; round up iff word < ceil(p * 2^32).
 *  - Blocks whose scale is zero (amax_b == 0, NV sb == 0) get codes +0.
 *
 * Scale-factor layouts:
 *  - FP4_SF_ROWMAJOR: [out_rows, L/block] bytes, row-major.
 *  - FP4_SF_MMA: the layout the block-scaled tensor-core MMA consumes: rows
 *    padded to 128 and k-groups to 4 (pads written as 0), 128x4 tiles stored
 *    with the k-tile index fastest, tile (rb,kb) at byte ((rb*G4)+kb)*512 and
 *    row r / k-group g inside it at (r%32)*16 + (r/32)*4 + g.  fp4_gemm reads
 *    only this layout.
 *
 * Conventions for every entry point:
 *  - All data pointers are DEVICE pointers (cudaMalloc'd or torch-owned) on
 *    the current device; the caller allocates and owns every buffer.  The
 *    library holds one small per-device scratch buffer (tensor-amax partials
 *    and a device error word), allocated on first use and kept until exit.
 *  - `stream` is a cudaStream_t owned by the caller (NULL = legacy default
 *    stream).  Every call is asynchronous on it; none synchronizes, except
 *    fp4_check_device_errors.
 *  - Argument, shape and alignment errors return a negative fp4_status before
 *    anything is launched.  A failed launch returns FP4_ERR_CUDA.  Nothing
 *    aborts, prints or throws across the ABI.  Calls that compute a tensor
 *    scale share the per-device scratch: two such calls that overlap in time
 *    on different streams of one device race.
 *  - Quantized tensors: axis = 1 quantizes along columns of x[rows, cols]
 *    (codes [rows, cols/2], scales per row); axis = 0 quantizes along rows
 *    and writes the transpose (codes [cols, rows/2]), so that the packed axis
 *    is always the contraction axis of fp4_gemm.  "out_rows" and "L" below
 *    are (rows, cols) for axis 1 and (cols, rows) for axis 0.
 *
 * Supported (format, block): (FP4_MXFP4, 32), (FP4_NVFP4, 16).
 */
#ifndef FP4_H_
#define FP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int fp4_status;
enum {
  FP4_OK = 0,
  FP4_ERR_ARG = -1,          /* null pointer, bad enum value, size not positive
                                (empty tensors are rejected, nothing launched)    */
  FP4_ERR_SHAPE = -2,        /* size not a multiple of what the format needs     */
  FP4_ERR_ALIGN = -3,        /* pointer or leading dimension misaligned          */
  FP4_ERR_UNSUPPORTED = -4,  /* (format, block) or option combination not built  */
  FP4_ERR_CUDA = -5,         /* CUDA runtime error at launch or set-up           */
  FP4_ERR_TIMEOUT = -6       /* a bounded device wait expired (reported later by
                                fp4_check_device_errors)                           */
};

enum { FP4_MXFP4 = 0, FP4_NVFP4 = 1 };              /* fp4_format    */
/* Quantizer-only format: NVFP4 codes and E4M3 scales whose block scale is, per
 * block, the one of max->6 (standard) and max->4 with the lower round-to-nearest
 * squared error ("Four Over Six: More Accurate NVFP4 Quantization with Adaptive
 * Block Scaling", Abstract; error in fp64, terms added in element order, ties
 * keep max->6).  Accepted by fp4_quantize and fp4_hadamard_quantize with block
 * 16; their outputs are plain NVFP4 (dequantize and GEMM with FP4_NVFP4). */
enum { FP4_NVFP4_4O6 = 2 };
/* Quantizer-only format: MXFP4 codes and E8M0 scales whose block exponent is
 * the smallest one whose grid reaches 7.25 * 2^E >= amax_b instead of the OCP
 * rule floor(log2 amax_b) - 2 (which clips up to 8 * 2^E): the MSE-fitted fixed
 * grid scale for MXFP4 with Hadamard rotations (summary post of "Bridging the
 * Gap Between Promise and Performance for Microscaling FP4 Quantization",
 * MR-GPTQ list item 1; 7.25 minimises the RTN squared error of rotated Gaussian
 * data over a 1/16 grid of [6, 8]).  Accepted by fp4_quantize and
 * fp4_hadamard_quantize with block 32; outputs are plain MXFP4. */
enum { FP4_MXFP4_GS = 3 };
enum { FP4_RTN = 0, FP4_SR = 1 };                   /* fp4_round     */
enum { FP4_SF_ROWMAJOR = 0, FP4_SF_MMA = 1 };       /* fp4_sf_layout */
enum { FP4_OUT_F32 = 0, FP4_OUT_BF16 = 1 };         /* fp4_dtype     */

/*
 * fp4_quantize -- block-scaled FP4 quantization of a bf16 matrix
 * ("FP4 All the Way", Abstract: NVFP4 blocks of 16 E2M1 with an E4M3 scale,
 * RTN forward / SR backward; "Bridging the Gap", Abstract: MXFP4
 * power-of-two scales).
 *
 *   x          bf16 [rows, cols], row stride `ld` elements (ld >= cols).
 *              16-byte aligned; cols and ld multiples of 8.
 *   fmt,block  (FP4_MXFP4, 32), (FP4_NVFP4, 16), (FP4_NVFP4_4O6, 16) or
 *              (FP4_MXFP4_GS, 32).
 *   axis       1: blocks along cols (cols % block == 0);
 *              0: blocks along rows (rows % block == 0), output transposed.
 *   rnd, seed  FP4_RTN, or FP4_SR with the 64-bit Philox key `seed`.
 *   tensor_scale_in   NV only, nullable, device fp32: use this s_t.
 *   tensor_scale_out  NV only, device fp32: receives the s_t used (may equal
 *              tensor_scale_in).  Required for NV, ignored for MX.
 *   codes      uint8 [out_rows, L/2], 16-byte aligned.
 *   scales     uint8, fp4_scales_bytes(...) bytes in layout `sf_layout`.
 * NV without tensor_scale_in launches an amax pass over x first.
 */
fp4_status fp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld,
                        int fmt, int block, int axis, int rnd, uint64_t seed,
                        const float* tensor_scale_in, float* tensor_scale_out,
                        uint8_t* codes, uint8_t* scales, int sf_layout, void* stream);

/*
 * fp4_quantize_shard -- fp4_quantize of a row shard: x holds rows
 * [first_row, first_row + rows) of a larger [*, cols] tensor, and the result is
 * those rows of the whole tensor's quantization ("FP4 All the Way", Abstract:
 * FP4 training across many accelerators, with stochastic rounding in the
 * backward pass).  Stochastic rounding draws the Philox words of the elements'
 * row-major indices in the whole tensor, (first_row + r) * cols + c, so shards
 * quantized on different devices concatenate to the unsharded codes bit for
 * bit.  For NVFP4 pass the whole tensor's scale in tensor_scale_in (e.g. from a
 * max all-reduce of the shards' fp4_amax and fp4_nv_tensor_scale); without it
 * the shard's own amax sets s_t.
 *   first_row  0 <= first_row < 2^40 (FP4_ERR_ARG otherwise); a multiple of the
 *              block for axis = 0 (FP4_ERR_SHAPE otherwise), so the shard's blocks
 *              are the tensor's.
 *   others     as fp4_quantize (first_row = 0 is fp4_quantize).
 */
fp4_status fp4_quantize_shard(const void* x, int64_t rows, int64_t cols, int64_t ld, int64_t first_row,
                              int fmt, int block, int axis, int rnd, uint64_t seed,
                              const float* tensor_scale_in, float* tensor_scale_out,
                              uint8_t* codes, uint8_t* scales, int sf_layout, void* stream);

/*
 * fp4_hadamard_quantize -- fp4_quantize with a block-diagonal Hadamard
 * rotation applied along the quantization axis first ("Bridging the Gap",
 * Abstract: block-wise Hadamard computed online for the activations; its
 * summary post, item 3: block-diagonal rotations).  Rotation: contiguous
 * blocks of `had_block` in {16, 32, 64, 128}, Sylvester order, scaled by
 * 1/sqrt(had_block), in fp32 in registers.  axis = 1 only; cols must be a
 * multiple of had_block.  rotated_out (nullable) receives the fp32 rotated
 * values [rows, cols] (row stride cols) for testing.
 */
fp4_status fp4_hadamard_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                 int fmt, int block, int axis, int rnd, uint64_t seed,
                                 const float* tensor_scale_in, float* tensor_scale_out,
                                 uint8_t* codes, uint8_t* scales, int sf_layout,
                                 int had_block, float* rotated_out, void* stream);

/*
 * fp4_quantize_dequantize -- fp4_quantize along axis 1 that also writes the
 * dequantized values ("FP4 All the Way", Abstract: the E2M1 values times their
 * block scale), as fp4_dequantize would compute them from the codes just
 * written, without re-reading the codes: one launch for quantize + dequantize.
 *   x .. sf_layout  as fp4_quantize with axis = 1 (fmt FP4_MXFP4, FP4_MXFP4_GS
 *              or FP4_NVFP4; FP4_NVFP4_4O6 is not supported here).
 *   out        fp32 or bf16 (out_dtype) [rows, cols], row stride cols,
 *              16-byte aligned.
 */
fp4_status fp4_quantize_dequantize(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                   int fmt, int block, int rnd, uint64_t seed,
                                   const float* tensor_scale_in, float* tensor_scale_out,
                                   uint8_t* codes, uint8_t* scales, int sf_layout,
                                   void* out, int out_dtype, void* stream);

/*
 * fp4_quantize_2d -- square-tile block quantization of a matrix
 * ("Pretraining Large Language Models with NVFP4", Abstract: a two-dimensional
 * quantization gives weights one consistent representation in the forward and
 * backward passes).  A block x block tile (16 x 16 NVFP4, 32 x 32 MXFP4)
 * shares one scale, computed from the tile's amax as fp4_quantize computes a
 * block's; each element is scaled and rounded once (SR: Philox word of its
 * row-major index in x), so W's codes along its rows and W^T's codes along its
 * rows are the same codes transposed, every segment carrying its tile's scale.
 *   x          bf16 [rows, cols], row stride ld; rows and cols multiples of the
 *              block; alignment as fp4_quantize.
 *   fmt,block,rnd,seed,tensor_scale_in,tensor_scale_out,sf_layout
 *              as fp4_quantize (NV without tensor_scale_in runs an amax pass).
 *   codes, scales      W along its rows: as fp4_quantize axis 1 (required).
 *   codes_t, scales_t  W^T along its rows, i.e. x quantized along axis 0:
 *              as fp4_quantize axis 0 ([cols, rows/2], 16-byte aligned); both
 *              null to skip, or both given.
 */
fp4_status fp4_quantize_2d(const void* x, int64_t rows, int64_t cols, int64_t ld,
                           int fmt, int block, int rnd, uint64_t seed,
                           const float* tensor_scale_in, float* tensor_scale_out,
                           uint8_t* codes, uint8_t* scales, uint8_t* codes_t, uint8_t* scales_t,
                           int sf_layout, void* stream);

/*
 * fp4_quantize_mse -- NVFP4 quantization with MSE-searched scales (summary
 * post of "Bridging the Gap Between Promise and Performance for Microscaling
 * FP4 Quantization", MR-GPTQ list item 1: the grid is fitted to the data by
 * optimizing it alternately per block and per tensor).
 *   Block step (tensor scale s fixed): each 16-element block takes, among its
 *   standard E4M3 byte b6 and the eight bytes below and above it (within
 *   1..126), the one whose round-to-nearest result has the least squared error
 *   (fp64, terms in element order; ties to the byte met first in the order
 *   b6, b6-1, b6+1, b6-2, ...); a block with b6 = 0 keeps 0.
 *   Tensor step: s becomes the best of fp32(s * (1 + k/64)), k = -8..8, each
 *   scored after its own block step by sum over blocks of
 *   floor(err_b * 2^(80 - 2 floor(log2 amax))) (an exact integer sum; ties to
 *   the smallest |k|, then k < 0).
 *   Schedule: s = amax / 2688, `iters` tensor steps (0..8), then a block step
 *   whose bytes quantize the codes with `rnd` (FP4_SR: Philox as fp4_quantize).
 *   fmt, block FP4_NVFP4, 16 (FP4_MXFP4: FP4_ERR_UNSUPPORTED).  Blocks run
 *              along cols (axis 1); cols % 16 == 0; x finite.
 *   x, rows, cols, ld, seed, codes, scales, sf_layout  as fp4_quantize axis 1.
 *   tensor_scale_out  device fp32, required: receives the searched s_t.
 * Outputs are plain NVFP4 (dequantize and GEMM with FP4_NVFP4).  Launches an
 * amax pass, `iters` tensor steps and the final quantize kernel; uses the
 * library's per-device scratch, so calls on one device must not run
 * concurrently on different streams.
 */
fp4_status fp4_quantize_mse(const void* x, int64_t rows, int64_t cols, int64_t ld,
                            int fmt, int block, int rnd, uint64_t seed, int iters,
                            float* tensor_scale_out, uint8_t* codes, uint8_t* scales,
                            int sf_layout, void* stream);

/*
 * fp4_dequantize -- codes + scales (+ s_t) back to floating point
 * ("FP4 All the Way", Abstract: the E2M1 values times their block scale).
 * MX: G[c] * 2^(b-127), exact in fp32.  NV: fp32(fp32(G[c] * sb) * s_t).
 *   codes  uint8 [rows, cols/2] (rows, cols = out_rows, L of the quantizer),
 *          16-byte aligned; out 16-byte aligned
 *   scales in `sf_layout`; tensor_scale device fp32 (NV), ignored for MX.
 *   out    fp32 or bf16 (RNE of the fp32 value) [rows, cols], row stride cols.
 */
fp4_status fp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                          int64_t rows, int64_t cols, int fmt, int block, int sf_layout,
                          void* out, int out_dtype, void* stream);

/*
 * fp4_gemm -- block-scaled FP4 x FP4 GEMM with fp32 accumulation on the
 * tcgen05 tensor cores ("Bridging the Gap", Abstract: FP4 GEMM on B200;
 * "Oscillation-Reduced MXFP4 Training", Abstract: MX matmuls on Blackwell);
 * M = 1 (one activation row, decoding) runs on the CUDA cores instead, with
 * exact per-block sums and one fp32 rounding per block.
 *   Y[M,N] = alpha * sum_k a[m,k] * b[n,k],  alpha = 1 (MX) or *a_ts * *b_ts (NV)
 *   a     uint8 codes [M, K/2] (K-major), a_sf scales in FP4_SF_MMA layout
 *   b     uint8 codes [N, K/2] (K-major), b_sf scales in FP4_SF_MMA layout
 *   a_ts, b_ts  device fp32 tensor scales (NV), ignored for MX
 *   y     fp32 or bf16 [M, N] with row stride ldy elements (ldy >= N)
 * K must be a multiple of 64 (K/2 bytes a multiple of 32); a, b, a_sf, b_sf
 * 16-byte aligned; y aligned to its element size (rows whose byte pitch and
 * base are 16-byte aligned get 128-bit stores); M, N >= 1 arbitrary.  Uses cudaGetDriverEntryPoint once to find
 * cuTensorMapEncodeTiled.
 */
fp4_status fp4_gemm(const uint8_t* a, const uint8_t* a_sf, const float* a_ts,
                    const uint8_t* b, const uint8_t* b_sf, const float* b_ts,
                    int64_t M, int64_t N, int64_t K, int fmt, int block,
                    void* y, int64_t ldy, int y_dtype, void* stream);

/*
 * fp4_gemm_quantize -- the block-scaled FP4 GEMM whose epilogue emits the next
 * layer's FP4 operand instead of Y ("Bridging the Gap", Abstract: FP4 kernels
 * with the activations' transforms computed online, here applied across
 * layers): Y = alpha * A . B^T as fp4_gemm computes it (fp32 accumulation,
 * the fp32 value fp4_gemm would store), quantized along its rows -- the next
 * GEMM's contraction axis -- with fp4_quantize's arithmetic, and never written.
 *   a .. fmt, block   as fp4_gemm (operands).
 *   out_fmt, out_block  (FP4_MXFP4, 32), (FP4_MXFP4_GS, 32) or (FP4_NVFP4, 16).
 *   rnd, seed   FP4_RTN, or FP4_SR with Philox words of Y's row-major element
 *               index (as fp4_quantize of a materialised Y[M, N]).
 *   out_tensor_scale  NVFP4 output: device fp32 s_t to quantize under (required;
 *               the amax of Y is not known until the GEMM ends, e.g. the
 *               previous step's scale); ignored for MXFP4.
 *   out_codes  uint8 [M, N/2], 16-byte aligned; out_scales in out_sf_layout
 *              (FP4_SF_MMA feeds the next fp4_gemm directly).
 * N must be a multiple of 32, K of 64.  Runs the single-SM or SM-pair GEMM
 * kernels (never the split-K clusters).
 */
fp4_status fp4_gemm_quantize(const uint8_t* a, const uint8_t* a_sf, const float* a_ts,
                             const uint8_t* b, const uint8_t* b_sf, const float* b_ts,
                             int64_t M, int64_t N, int64_t K, int fmt, int block,
                             int out_fmt, int out_block, int rnd, uint64_t seed,
                             const float* out_tensor_scale, uint8_t* out_codes,
                             uint8_t* out_scales, int out_sf_layout, void* stream);

/*
 * fp4_amax -- max |x| over a bf16 matrix into one device fp32 (the first
 * pass of NVFP4's per-tensor scale, "FP4 All the Way", Abstract).  Used when
 * a tensor is sharded and the maxima are combined across ranks before
 * fp4_nv_tensor_scale.  Same x requirements as fp4_quantize.
 */
fp4_status fp4_amax(const void* x, int64_t rows, int64_t cols, int64_t ld,
                    float* amax_out, void* stream);

/*
 * fp4_amax_noalloc -- the same max |x| as fp4_amax, for callers that must not
 * allocate device memory.  (The pages describe nothing like it; it exists for
 * deployment.)  Callers that cannot call cudaMalloc include a process whose
 * caching allocator already owns all free device memory, a latency-critical
 * path that cannot absorb the synchronization an allocation may cause, and
 * code running inside an allocator callback, which must not re-enter the CUDA
 * allocator.  fp4_amax allocates its scratch on first use; this entry point
 * never calls cudaMalloc, cudaFree or any allocating routine.
 *   Scratch: a fixed 33,024-byte array inside libfp4 (partial maxima of up to
 *   8192 CTAs plus a counter), held by every GPU that loads the library until
 *   the process exits.  One CTA covers 8192 elements, so inputs are limited to
 *   rows * cols <= 2^26 (67,108,864) elements; larger inputs return
 *   FP4_ERR_SHAPE.  Other requirements and errors as fp4_amax.
 *   Set-up: the first call on each device (and the first after that device's
 *   context was destroyed and created again, e.g. by cudaDeviceReset), made
 *   with that device current, loads the library's amax kernel and looks up
 *   the array's device address (cudaGetSymbolAddress).  Under CUDA's lazy
 *   module loading this is where the kernel's code and the array first take
 *   device memory, so the first call can fail with FP4_ERR_CUDA when no device
 *   memory is left.  Make it early, as a warm-up (e.g. on a tiny tensor): before
 *   a caching allocator takes all free memory, outside any allocator callback
 *   and before any stream capture.  Later calls take no device memory.
 *   Every call resets the counter, and all calls share the one array: calls
 *   that overlap on the GPU (e.g. on two streams) race, so the caller must
 *   serialize them (one stream, or events between the streams).
 */
fp4_status fp4_amax_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld,
                            float* amax_out, void* stream);

/* fp4_nv_tensor_scale -- s_t = fp32(amax / 2688), 1.0 for amax == 0, on the
 * device (one thread).  amax and tensor_scale_out are device fp32 pointers. */
fp4_status fp4_nv_tensor_scale(const float* amax, float* tensor_scale_out, void* stream);

/* Bytes of packed codes for a [rows, cols] input (either axis). */
size_t fp4_codes_bytes(int64_t rows, int64_t cols);
/* Bytes of scales for a [rows, cols] input quantized along `axis`; 0 on bad arguments. */
size_t fp4_scales_bytes(int64_t rows, int64_t cols, int block, int axis, int sf_layout);

/* Synchronizes `stream`, then reads and clears the device error word that
 * bounded waits set; returns FP4_ERR_TIMEOUT if any wait expired since the
 * last check, FP4_ERR_CUDA on a runtime error, else FP4_OK. */
fp4_status fp4_check_device_errors(void* stream);

/* Static string for a status code. */
const char* fp4_status_string(fp4_status status);

#ifdef __cplusplus
}
#endif
#endif /* FP4_H_ */
