/*
 * hq.h -- C ABI of libhq.so: hybrid BF16/Int4 compression of tensor-parallel partial sums on
 * NVIDIA B200 (sm_100a).
 *
 * The method is the one summarised on the page "Revolutionizing LLM Inference: The Power of
 * Efficient Low-Bit Communication" (about "Towards Efficient Low-Bit Communication for Tensor
 * Parallel LLM Inference"):
 *   - section "Combating Quantization Errors with Tensor Parallelism": each rank's partial sum
 *     is quantized *before* the ranks synchronise, so the per-rank errors add up around zero;
 *   - section "The Hybrid Quantization Algorithm": Calibration (per-feature moving averages of
 *     the observed min and max on each device), Selection of High Precision Features (rank
 *     features by quantization range, keep the top ones in BF16), Inference (the rest go to
 *     4 bits; after communication everything is converted back and summed across devices).
 * The page gives no formula, bit layout or interface; the exact arithmetic below is a stated
 * reading of it (the readings are numbered R1..R19 where they are used).
 *
 * Notation: P ranks, T rows (tokens), H features (columns), k features kept in BF16, H' = H - k.
 * One GPU simulates the P ranks: a tensor [P][T][H] holds every rank's partial sum, and the
 * per-rank semantics are the same as for one real rank calling with P = 1 on its own slice.
 *
 * Conventions for every call:
 *   - All arrays are dense, row-major, in device memory, owned by the caller.  The library
 *     allocates nothing and keeps no state between calls (apart from one device error word, see
 *     hq_read_device_error, cached launch facts per device, and the self-test setting of
 *     hq_selftest_set_pipeline_stall).  bf16 values are passed as their uint16_t bit patterns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Every call
 *     only enqueues work on it and returns; results are ready when the stream reaches them.
 *   - Arguments are checked on the host before anything is enqueued.  On a bad argument the
 *     call returns HQ_ERR_INVALID_ARG or HQ_ERR_MISALIGNED and enqueues nothing.  A failed
 *     launch returns HQ_ERR_CUDA.
 *   - Shape limits: 1 <= P <= 64; 8 <= H <= 32768 with H % 8 == 0; 0 <= k <= H with k % 8 == 0.
 *     A pointer to an array that is empty for the given sizes (keep_idx/side when k == 0,
 *     rest_idx/codes when k == H, every per-row array when T == 0) may be NULL.
 *   - Alignment: x, side, out, ema_min, ema_max, scale, inv_scale and zero 16 bytes; codes,
 *     keep_idx and rest_idx 4 bytes.
 *   - keep_idx must be strictly ascending with values in [0, H) and rest_idx must be its
 *     ascending complement, as hq_select_topk writes them.  The kernels read every index
 *     through range checks: an index outside [0, H) is not dereferenced, and the first one seen
 *     sets the device error word to HQ_ERR_BAD_INDEX (the outputs are then unspecified).
 *   - Outputs must not overlap inputs.
 */
#ifndef HQ_H
#define HQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HQ_OK = 0,
  HQ_ERR_INVALID_ARG = 1, /* a size, count, decay or NULL pointer outside the rules above   */
  HQ_ERR_MISALIGNED = 2,  /* a pointer below its required alignment                          */
  HQ_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed                     */
  HQ_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up (device error word)          */
  HQ_ERR_BAD_INDEX = 5    /* a kernel met an index outside [0, H) (device error word)        */
} hq_status;

typedef enum { HQ_OUT_BF16 = 0, HQ_OUT_F32 = 1 } hq_out_dtype;

/*
 * Calibration -- section "The Hybrid Quantization Algorithm", bullet "Calibration".
 * Folds one calibration batch into the per-rank, per-feature moving averages of min and max
 * (R1, R2): for each rank r and feature h, bmin/bmax = min/max over the batch's T rows of
 * x[r][t][h] (NaN values are skipped; a result of -0 is stored as +0), then
 *   first_batch != 0:  ema_min = bmin,  ema_max = bmax;
 *   otherwise:         ema = beta*ema + (1-beta)*b, each product and the sum rounded to fp32,
 *                      with (1-beta) itself computed in fp32.
 *   x        bf16 [P][T][H], T >= 1
 *   beta     decay, 0 <= beta < 1
 *   ema_min, ema_max  float [P][H], read (unless first_batch) and written
 */
hq_status hq_calibrate(const uint16_t* x, int P, int T, int H, float beta, int first_batch,
                       float* ema_min, float* ema_max, void* stream);

/*
 * Selection -- section "The Hybrid Quantization Algorithm", bullet "Selection of High
 * Precision Features", with the 4-bit grid of bullet "Calibration" (R3, R4, R5, R14).
 * For every rank and feature: lo = min(ema_min, 0), hi = max(ema_max, 0),
 *   scale = (hi - lo)/15, inv_scale = 1/scale (both correctly rounded fp32),
 *   zero  = clamp(rint(-lo * inv_scale), 0, 15)  (round half to even);
 *   a scale that is 0, subnormal, infinite or NaN gives scale = inv_scale = 1, zero = 0.
 * Score of a feature = sum over ranks, in rank order in fp32, of (hi - lo).  The k features with
 * the largest scores are kept in BF16 (equal scores: lower feature index first).
 *   ema_min, ema_max  float [P][H]
 *   keep_idx int32 [k]    the kept features, ascending
 *   rest_idx int32 [H-k]  all other features, ascending
 *   scale, inv_scale float [P][H], zero uint8 [P][H]  (computed for kept features too)
 * Two kernels on `stream`; between them keep_idx and rest_idx hold the scores (the library uses
 * no other memory), so they must not be read until the stream has passed the call.
 */
hq_status hq_select_topk(const float* ema_min, const float* ema_max, int P, int H, int k,
                         int32_t* keep_idx, int32_t* rest_idx, float* scale, float* inv_scale,
                         uint8_t* zero, void* stream);

/*
 * Quantize-pack, the sending side of bullet "Inference" (R6, R7).  For every rank r and row t:
 *   side[r][j][t]  = x[r][t][keep_idx[j]]                     (bf16 bits, unchanged)
 *   code of compact column c (feature h = rest_idx[c]):
 *     q = clamp(rint(x * inv_scale[r][h]) + zero[r][h], 0, 15), the product in fp32,
 *     round half to even; +-inf saturate to 15 / 0; NaN gives q = zero[r][h].
 *   codes[r][t][c/8] holds code c in bits 4*(c%8) .. 4*(c%8)+3.
 *   x     bf16 [P][T][H]      (T >= 0; T == 0 enqueues nothing)
 *   codes uint32 [P][T][H'/8] -- the wire buffer of the 4-bit part
 *   side  bf16 [P][k][T]      -- the wire buffer of the BF16 part, feature-major: the T rows of
 *                                kept feature j are contiguous
 */
hq_status hq_quantize_pack(const uint16_t* x, int P, int T, int H, int k, const int32_t* keep_idx,
                           const int32_t* rest_idx, const float* inv_scale, const uint8_t* zero,
                           uint32_t* codes, uint16_t* side, void* stream);

/*
 * Dequant-reduce, the receiving side of bullet "Inference": every rank's shard is converted back
 * and the ranks are summed in rank order (R9, R10, R11).  For row t:
 *   non-kept feature h = rest_idx[c]:  acc = +0;  for r = 0..P-1:
 *       acc = fma(float(q_r - zero[r][h]), scale[r][h], acc)      (one rounding per rank)
 *   kept feature h = keep_idx[j]:      acc = +0;  for r = 0..P-1:  acc = acc + side[r][j][t]
 *   out[t][h] = acc as fp32 (HQ_OUT_F32), or rounded to bf16 nearest-even (HQ_OUT_BF16); a
 *   NaN sum is written as the canonical quiet NaN (0x7FC00000 / 0x7FC0).
 *   codes, side as written by hq_quantize_pack; out [T][H] of the chosen type.
 */
hq_status hq_dequant_reduce(const uint32_t* codes, const uint16_t* side, int P, int T, int H, int k,
                            const int32_t* keep_idx, const int32_t* rest_idx, const float* scale,
                            const uint8_t* zero, void* out, hq_out_dtype out_dtype, void* stream);

/*
 * Dequant-reduce of wires that lie in P separate buffers, one per rank: the receiving side of
 * bullet "Inference" reading every rank's wire where it lies, with no gathering copy first.
 * Between GPUs joined by NVLink/NVSwitch, codes[r] and side[r] can be another GPU's memory
 * mapped into this process (peer access, or a symmetric-memory mapping): each CTA then reads the
 * remote tiles it reduces over the interconnect with tensor-memory-accelerator loads (no
 * multicast), so the exchange of the wire and its reduction are one kernel ("Key Observations
 * and Future Directions" leaves the all-reduce algorithm open).  The caller orders every rank's
 * hq_quantize_pack before this call (e.g. a stream-ordered barrier across the ranks) and keeps
 * the buffers unchanged until it has completed.
 *   codes  host array of P device pointers; codes[r] uint32 [T][(H-k)/8], rank r's 4-bit wire
 *   side   host array of P device pointers; side[r] bf16 [k][T] (side may be NULL when k == 0)
 *   1 <= P <= 8; H - k a positive multiple of 32 (code rows of a multiple of 16 bytes);
 *   codes[r] and side[r] 16-byte aligned.
 * Parameters, output, arithmetic (R9-R11, rank order 0..P-1) and errors as in hq_dequant_reduce;
 * the result is bitwise that of hq_dequant_reduce on the stacked wire.
 */
hq_status hq_dequant_reduce_ranks(const uint32_t* const* codes, const uint16_t* const* side, int P, int T, int H,
                                  int k, const int32_t* keep_idx, const int32_t* rest_idx, const float* scale,
                                  const uint8_t* zero, void* out, hq_out_dtype out_dtype, void* stream);

/*
 * Dequant-reduce, literal reading of bullet "Inference" (R19): after communication each rank's
 * tensor is first made BF16 and the ranks' BF16 tensors are then combined.  Same arguments,
 * layouts, ownership and errors as hq_dequant_reduce; only non-kept features differ:
 *   non-kept feature h = rest_idx[c]:  acc = +0;  for r = 0..P-1:
 *       v = float(q_r - zero[r][h]) * scale[r][h]            (one fp32 product)
 *       acc = acc + bf16(v)          (v rounded to bf16, nearest-even, then added in fp32)
 * Kept features and the output are as in hq_dequant_reduce.  Used to measure what the extra
 * per-rank rounding costs in accuracy (the selection ablation); the default reading keeps each
 * rank's exact product.
 */
hq_status hq_dequant_reduce_bf16_shards(const uint32_t* codes, const uint16_t* side, int P, int T, int H,
                                        int k, const int32_t* keep_idx, const int32_t* rest_idx,
                                        const float* scale, const uint8_t* zero, void* out,
                                        hq_out_dtype out_dtype, void* stream);

/*
 * Fused compress-reduce (section "Combating Quantization Errors with Tensor Parallelism": the
 * partial sums are quantized and then summed): out equals hq_quantize_pack followed by
 * hq_dequant_reduce, bit for bit (R12), computed from x in one pass without a wire buffer.
 * If codes_or_null / side_or_null are not NULL the wire buffers are written too (by the
 * quantize-pack kernel, i.e. x is read a second time in that case).
 */
hq_status hq_compress_reduce(const uint16_t* x, int P, int T, int H, int k, const int32_t* keep_idx,
                             const int32_t* rest_idx, const float* scale, const float* inv_scale,
                             const uint8_t* zero, void* out, hq_out_dtype out_dtype,
                             uint32_t* codes_or_null, uint16_t* side_or_null, void* stream);

/*
 * Partial-channel synchronisation -- the abstract of "Communication-Aware Architecture for
 * Tensor-parallelism" (CAAT-Net) on the first page: tensor-parallel ranks can do without
 * synchronising every activation channel.  Reading R20: a block of consecutive features of each
 * rank's partial sum goes through the hybrid wire and the rank-ordered sum, and every rank keeps
 * its own partial sum in the other features.  The four calls below are the calls above on such a
 * block: `H` is the block's width, x points at the block's first feature of rank 0, row 0, and
 * rows are ldx elements apart (rank r's rows start at x + r*T*ldx); out points at the block's
 * first feature of row 0 and its rows are ldo elements apart.  Only the block's columns of out
 * are written: a rank that keeps its own partial sum in out's other columns gets exactly the
 * reading's result.  Statistics, parameters, codes and side are those of the dense [P][T][H]
 * block (as if it were copied out first), so hq_select_topk and hq_wire_bytes_per_row apply as
 * they are, and a rank sends (H-k)/2 + 2k bytes per row for the block alone.
 *   ldx, ldo  >= H and multiples of 8; x and out 16-byte aligned (so the block starts at a
 *             multiple of 8 features).  Other arguments, checks and errors as in the calls above.
 */
hq_status hq_calibrate_ld(const uint16_t* x, int ldx, int P, int T, int H, float beta, int first_batch,
                          float* ema_min, float* ema_max, void* stream);
hq_status hq_quantize_pack_ld(const uint16_t* x, int ldx, int P, int T, int H, int k, const int32_t* keep_idx,
                              const int32_t* rest_idx, const float* inv_scale, const uint8_t* zero,
                              uint32_t* codes, uint16_t* side, void* stream);
hq_status hq_dequant_reduce_ld(const uint32_t* codes, const uint16_t* side, int P, int T, int H, int k,
                               const int32_t* keep_idx, const int32_t* rest_idx, const float* scale,
                               const uint8_t* zero, void* out, int ldo, hq_out_dtype out_dtype, void* stream);
hq_status hq_compress_reduce_ld(const uint16_t* x, int ldx, int P, int T, int H, int k, const int32_t* keep_idx,
                                const int32_t* rest_idx, const float* scale, const float* inv_scale,
                                const uint8_t* zero, void* out, int ldo, hq_out_dtype out_dtype,
                                uint32_t* codes_or_null, uint16_t* side_or_null, void* stream);

/*
 * The two-step compressed all-reduce of P simulated ranks on one GPU -- the quantized
 * reduce-scatter then re-quantized all-gather of the "Flash Communication" abstract (third page),
 * reading R22 (no formula there).  Step 1: hq_quantize_pack and hq_dequant_reduce of x [P][T][H]
 * with the step-1 selection and grids, the reduced tensor rounded to bf16.  Step 2: reducer j owns
 * rows [j*T/P, (j+1)*T/P); it quantize-packs its block with row j of the step-2 grids
 * (scale2/inv_scale2/zero2 [P][H]) and the step-2 kept set (keep2 [k2], rest2 [H-k2]), and the
 * block is dequantized with the same grid (P = 1, nothing summed) into those rows of out.
 *   x, keep_idx .. zero   as in hq_compress_reduce (step 1)
 *   k2, keep2 .. zero2    the step-2 selection and the reducers' grids
 *   workspace             device memory of at least hq_two_step_workspace_bytes(P, T, H, k, k2)
 *                         bytes, 256-byte aligned, owned by the caller: it holds the step-1 wire,
 *                         the reduced tensor and the step-2 wires (its contents are scratch)
 *   out                   [T][H], bf16 or fp32
 *   T % P == 0 and H % 16 == 0 (every reducer's row of zero2 then starts on a 16-byte boundary).
 * Enqueues 4 kernels on `stream`: step 2's P blocks are one quantize-pack over P "ranks" of T/P
 * rows and one dequant-reduce launch over P independent one-rank problems (when H - k2 is not a
 * multiple of 32 its code rows cannot be staged by TMA, and that dequant is one launch per block).
 * Errors as in the calls above, all checked before anything is enqueued; a workspace that is NULL
 * or too small is HQ_ERR_INVALID_ARG, one below 256-byte alignment HQ_ERR_MISALIGNED.
 */
hq_status hq_two_step_reduce(const uint16_t* x, int P, int T, int H, int k, const int32_t* keep_idx,
                             const int32_t* rest_idx, const float* scale, const float* inv_scale, const uint8_t* zero,
                             int k2, const int32_t* keep2, const int32_t* rest2, const float* scale2,
                             const float* inv_scale2, const uint8_t* zero2, void* workspace, size_t workspace_bytes,
                             void* out, hq_out_dtype out_dtype, void* stream);

/* Bytes of workspace hq_two_step_reduce needs (0 for sizes it rejects). */
size_t hq_two_step_workspace_bytes(int P, int T, int H, int k, int k2);

/*
 * hq_two_step_reduce without a workspace argument: it allocates nothing and takes no memory from
 * the caller beyond its inputs and outputs.  (The pages have no counterpart: this is a service of
 * the library, not a step of the method.)  It is meant for callers that cannot call cudaMalloc --
 * a serving process whose device memory is fixed at start-up, a plugin running inside another
 * framework's memory pool, or a latency-critical loop where an allocation's device-wide
 * synchronisation is not acceptable.
 *
 * The scratch lives in a fixed array of HQ_TWO_STEP_NOALLOC_MAX_BYTES bytes in the global memory
 * of every GPU that loads the library, held until the process exits.  Problems whose
 * hq_two_step_workspace_bytes(P, T, H, k, k2) exceeds it (or is 0) return HQ_ERR_INVALID_ARG before
 * anything is enqueued: decode-size problems fit (P = 4, T = 32, H = 4096 needs under 1 MiB), the
 * prefill shapes need hq_two_step_reduce and a workspace of their own.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 *     that device current) and keeps it; make that first call before any stream capture.
 *   - Every call on a device shares the one array, and it keeps the last call's contents.  Nothing
 *     in it needs to start at zero: every byte a call reads, the same call has written first.
 *   - Calls whose work overlaps on the GPU (for example on two streams without an order between
 *     them) race on the array and give undefined results: order them.
 * Arguments, result and errors otherwise as in hq_two_step_reduce; the result is bitwise the same.
 */
#define HQ_TWO_STEP_NOALLOC_MAX_BYTES ((size_t)16 << 20)
hq_status hq_two_step_reduce_noalloc(const uint16_t* x, int P, int T, int H, int k, const int32_t* keep_idx,
                                     const int32_t* rest_idx, const float* scale, const float* inv_scale,
                                     const uint8_t* zero, int k2, const int32_t* keep2, const int32_t* rest2,
                                     const float* scale2, const float* inv_scale2, const uint8_t* zero2, void* out,
                                     hq_out_dtype out_dtype, void* stream);

/* A static string naming a status. */
const char* hq_status_string(hq_status s);

/*
 * Returns and clears the device error word of the current device: HQ_OK if no kernel recorded
 * an error since the last call, else the first recorded status (HQ_ERR_BAD_INDEX,
 * HQ_ERR_TIMEOUT).  The word is device-wide: kernels on every stream record into it.  The call
 * enqueues one single-thread kernel on `stream` that exchanges the word with 0 atomically, copies
 * the old value back and synchronises `stream`; so work ordered before it on `stream` has been
 * counted, and an error recorded concurrently by a kernel on another stream is counted by this
 * call or by the next one, never lost.  Calls from several host threads are serialised.  Returns
 * HQ_ERR_CUDA if the launch, the copy or the synchronisation fails.
 */
hq_status hq_read_device_error(void* stream);

/*
 * Self-test of the bounded waits used by the TMA pipelines (no counterpart on the page; it
 * exists so that failure detection can be tested without faulting or hanging a GPU): launches
 * one thread that waits on a shared-memory mbarrier nothing ever arrives on, giving up after
 * `limit_cycles` clock cycles.  It records HQ_ERR_TIMEOUT in the device error word (read it
 * with hq_read_device_error) and returns; the context stays usable.
 */
hq_status hq_selftest_bounded_wait(long long limit_cycles, void* stream);

/*
 * Self-test of the pipelines' abort path (no counterpart on the page; it exists so that failure
 * detection in the real TMA pipelines -- quantize-pack, dequant-reduce and compress-reduce -- can
 * be tested without faulting or hanging a GPU).  After hq_selftest_set_pipeline_stall(c, d) with
 * c > 0 and d > 0, every pipeline kernel launched by this process lets its producer lane idle for
 * d clock cycles before its first load, and bounds its consumers' waits by c cycles instead of
 * about a second.  With c well below d the consumers give up: the kernel records HQ_ERR_TIMEOUT,
 * raises its abort flag, the producer issues its first loads, sees the flag, waits (on the long
 * bound) for those loads to land, and the kernel returns with its outputs unspecified.
 * hq_selftest_set_pipeline_stall(0, 0) restores the normal bounds.  Process-wide; not for use
 * while other threads launch work.
 *   consumer_limit_cycles  >= 0;  producer_delay_cycles  0 .. 2^31 (about a second)
 * Returns HQ_ERR_INVALID_ARG if either is out of range or exactly one of them is 0.
 */
hq_status hq_selftest_set_pipeline_stall(long long consumer_limit_cycles, long long producer_delay_cycles);

/* Bytes of the two wire buffers per rank and row: 4-bit part (H-k)/2, BF16 part 2k. */
int64_t hq_wire_bytes_per_row(int H, int k);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H */
