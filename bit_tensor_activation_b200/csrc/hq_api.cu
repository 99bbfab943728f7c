// hq_api.cu -- the C ABI of libhq.so (declared in include/hq.h).
//
// One translation unit holds every kernel (so the device error word is a single symbol).  Each
// entry point checks its arguments on the host, picks a launch shape, enqueues one kernel on the
// caller's stream and returns; nothing is allocated and nothing waits, except
// hq_read_device_error, which synchronises the stream it is given.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <type_traits>
#include <mutex>

#include "hq.h"
#include "hq_common.cuh"
#include "hq_tma.cuh"
#include "k_calibrate.cuh"
#include "k_dequant.cuh"
#include "k_fused.cuh"
#include "k_quantize.cuh"
#include "k_select.cuh"

namespace {

constexpr int kMaxRanks = 64;
static_assert(kMaxRanks <= hq::kSelMaxRanks, "the parameter kernel stages one range per rank");
constexpr int kMaxDevices = 64;
constexpr long long kMaxStallDelayCycles = 1LL << 31;  // about a second

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

hq_status check_shape(int P, int H, int k) {
  if (P < 1 || P > kMaxRanks) return HQ_ERR_INVALID_ARG;
  if (H < 8 || H > hq::kMaxH || (H % 8) != 0) return HQ_ERR_INVALID_ARG;
  if (k < 0 || k > H || (k % 8) != 0) return HQ_ERR_INVALID_ARG;
  return HQ_OK;
}

// Resident CTAs per SM of one kernel for each rank count P (its shared memory grows with P),
// queried once per device; the kernel's dynamic shared-memory limit is raised to the largest size
// requested so far.
struct OccupancyCache {
  int smem_set = 0;
  int per_sm[kMaxRanks + 1] = {};
};

// Launch-shape facts cached per device: SM count and resident CTAs per SM of each kernel.
struct DeviceInfo {
  int sms = 0;
  int qt_blocks = 0;
  bool select_smem_set = false;
  OccupancyCache dequant_tma[2][2];  // [fp32 out][bf16 shards]
  OccupancyCache dequant_cp[2][2];
  OccupancyCache fused[2];           // [fp32 out]
};

// cuTensorMapEncodeTiled, fetched once through the runtime (no link-time libcuda dependency).
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_encode_mu;

bool get_encode() {
  std::lock_guard<std::mutex> lock(g_encode_mu);
  if (g_encode) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return false;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

// Row-major 2-D tensor [rows][cols] of `elem`-byte elements (row pitch `pitch` bytes, cols*elem
// when 0; a multiple of 16) read in boxes of box_rows x box_cols; out-of-range box elements read as 0.
bool encode_2d(CUtensorMap* map, const void* base, CUtensorMapDataType type, size_t elem, uint64_t cols,
               uint64_t rows, uint32_t box_cols, uint32_t box_rows,
               CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B, uint64_t pitch = 0) {
  if (!get_encode()) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch ? pitch : cols * elem};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(map, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

hq_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.sms == 0) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return HQ_ERR_CUDA;
    const int qt_smem = (int)(sizeof(hq::QtSmem) + 128);
    if (cudaFuncSetAttribute(hq::quantize_pack_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             qt_smem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.qt_blocks, hq::quantize_pack_tma_kernel,
                                                      hq::kQtThreads, qt_smem) != cudaSuccess)
      return HQ_ERR_CUDA;
    if (d.qt_blocks < 1) d.qt_blocks = 1;
  }
  *out = &d;
  return HQ_OK;
}

hq_status launched() { return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA; }

// CTAs of `kern` resident per SM with `smem` bytes of dynamic shared memory (at least 1), from the
// device's cache; the first use for a P sets the shared-memory limit and runs the query.
template <typename Kernel>
hq_status occupancy(OccupancyCache& c, Kernel kern, int threads, size_t smem, int P, int* per_sm) {
  std::lock_guard<std::mutex> lock(g_dev_mu);
  if (c.per_sm[P] == 0) {
    if ((int)smem > c.smem_set) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return HQ_ERR_CUDA;
      c.smem_set = (int)smem;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem) != cudaSuccess) return HQ_ERR_CUDA;
    c.per_sm[P] = n < 1 ? 1 : n;
  }
  *per_sm = c.per_sm[P];
  return HQ_OK;
}

// Wait bounds of the pipeline kernels.  Normal launches use the long default everywhere; the
// abort self-test (hq_selftest_set_pipeline_stall) shortens the consumers' bound and delays the
// producers' first loads.
std::atomic<long long> g_stall_consumer_limit{0};
std::atomic<long long> g_stall_producer_delay{0};

hq::WaitLimits wait_limits() {
  const long long c = g_stall_consumer_limit.load(), d = g_stall_producer_delay.load();
  if (c == 0 && d == 0) return hq::WaitLimits{hq::kWaitLimitCycles, hq::kWaitLimitCycles, 0};
  return hq::WaitLimits{c, hq::kWaitLimitCycles, d};
}

long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }

// One wave of `resident` CTAs over S slices of nb_all row blocks each: every slice gets `base`
// row chunks and slices 0..extra-1 one more; never more chunks than blocks, at least one.
struct WaveChunks {
  int base, extra;
};
WaveChunks wave_chunks(long long resident, int S, long long nb_all) {
  long long base = resident / S, extra = resident - base * S;
  if (base < 1) base = 1, extra = 0;
  if (base >= nb_all) base = std::max(nb_all, 1LL), extra = 0;
  return WaveChunks{(int)base, (int)extra};
}

// Slices x row chunks of the cp.async dequant-reduce kernel: one wave of CTAs at most.
void slice_chunks(int T, int S, long long resident, int rows_per_block, int* chunks, int* rows_per_chunk) {
  long long c = resident / S;
  if (c < 1) c = 1;
  const long long max_c = ceil_div(T, rows_per_block);
  if (c > max_c) c = max_c;
  long long rpc = ceil_div(ceil_div(T, c), rows_per_block) * rows_per_block;
  *rows_per_chunk = (int)rpc;
  *chunks = (int)ceil_div(T, rpc);
}

// Where dequant-reduce reads the P ranks' wires: one stacked buffer [P][T][W] / [P][k][T], or one
// buffer per rank (host arrays of P device pointers; each may be a peer GPU's memory).
struct WireSrc {
  const uint32_t* codes = nullptr;
  const uint16_t* side = nullptr;
  const uint32_t* const* codes_r = nullptr;
  const uint16_t* const* side_r = nullptr;
  bool per_rank = false;
};

// nbatch > 1: nbatch independent problems of P ranks each, stacked (problem b: ranks b*P .. b*P+P-1
// of the wire and the parameters, output rows b*T .. b*T+T-1); one launch when TMA can stage them.
template <typename OutT, bool kShard>
hq_status launch_dequant(const WireSrc& src, int P, int T, int H, int k, const int32_t* keep_idx, const float* scale,
                         const uint8_t* zero, void* out, int ldo, cudaStream_t st, DeviceInfo& d, int nbatch = 1) {
  const int S = (H + 8 * hq::kDqSliceGroups - 1) / (8 * hq::kDqSliceGroups);
  const int Wr = (H - k) / 8;
  hq::DqWire wire;
  memset(&wire, 0, sizeof wire);
  wire.per_rank = src.per_rank ? 1 : 0;
  bool tma = Wr >= 4 && Wr % 4 == 0;
  // side[r][j][t] as [k][T] rows: boxes of 32 rows (inner) x 32 kept features; needs rows of a
  // multiple of 16 bytes (T % 8 == 0), else the kept sums read the side buffer directly
  bool side_tma = k > 0 && T % 8 == 0;
  if (!src.per_rank) {
    tma = tma && aligned(src.codes, 16) &&
          encode_2d(&wire.code[0], src.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)Wr,
                    (uint64_t)nbatch * P * T, hq::kDtWords, hq::kDtTileRows);
    side_tma = tma && side_tma &&
               encode_2d(&wire.side[0], src.side, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)T,
                         (uint64_t)nbatch * P * k, hq::kDtTileRows, hq::kDtSideCols, CU_TENSOR_MAP_L2_PROMOTION_NONE);
  } else {
    for (int r = 0; r < P && tma; ++r)
      tma = encode_2d(&wire.code[r], src.codes_r[r], CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)Wr, (uint64_t)T,
                      hq::kDtWords, hq::kDtTileRows);
    for (int r = 0; r < P && side_tma; ++r)
      side_tma = encode_2d(&wire.side[r], src.side_r[r], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)T, (uint64_t)k,
                           hq::kDtTileRows, hq::kDtSideCols, CU_TENSOR_MAP_L2_PROMOTION_NONE);
    for (int r = 0; r < P; ++r) wire.side_ptr[r] = k > 0 ? src.side_r[r] : nullptr;
    if (!tma || nbatch != 1) return HQ_ERR_INVALID_ARG;  // per-rank buffers: TMA kernel, one problem
    side_tma = side_tma && tma;
  }
  constexpr int kF32 = std::is_same<OutT, float>::value ? 1 : 0;
  if (tma) {
    const size_t smem = hq::dt_smem_bytes(P);
    auto kern = hq::dequant_reduce_tma_kernel<OutT, kShard>;
    int per_sm = 0;
    if (occupancy(d.dequant_tma[kF32][kShard], kern, hq::kDtThreads, smem, P, &per_sm) != HQ_OK) return HQ_ERR_CUDA;
    // one wave that fills every resident CTA slot (wave_chunks)
    const long long nb_all = ceil_div(T, hq::kDtTileRows);
    const WaveChunks wc = wave_chunks((long long)d.sms * per_sm / nbatch, S, nb_all);
    const dim3 grid((unsigned)(S * wc.base + wc.extra), (unsigned)nbatch);
    kern<<<grid, hq::kDtThreads, smem, st>>>(wire, side_tma ? 1 : 0, src.side, P, T, H, k, keep_idx, scale, zero,
                                             static_cast<OutT*>(out), ldo, S, wc.base, wc.extra, wait_limits());
    return launched();
  }
  if (nbatch > 1) {  // the cp.async kernel takes one problem per launch
    const int Wr2 = (H - k) / 8;
    for (int b = 0; b < nbatch; ++b) {
      WireSrc one;
      one.codes = src.codes ? src.codes + (size_t)b * P * T * Wr2 : nullptr;
      one.side = src.side ? src.side + (size_t)b * P * k * T : nullptr;
      const hq_status r = launch_dequant<OutT, kShard>(one, P, T, H, k, keep_idx, scale + (size_t)b * P * H,
                                                       zero + (size_t)b * P * H,
                                                       static_cast<OutT*>(out) + (size_t)b * T * ldo, ldo, st, d, 1);
      if (r != HQ_OK) return r;
    }
    return HQ_OK;
  }
  const size_t smem = hq::dq_smem_bytes(P);
  auto kern = hq::dequant_reduce_kernel<OutT, kShard>;
  int per_sm = 0;
  if (occupancy(d.dequant_cp[kF32][kShard], kern, hq::kDqThreads, smem, P, &per_sm) != HQ_OK) return HQ_ERR_CUDA;
  int chunks, rpc;
  slice_chunks(T, S, (long long)d.sms * per_sm, hq::kDqR, &chunks, &rpc);
  kern<<<(unsigned)(S * chunks), hq::kDqThreads, smem, st>>>(src.codes, src.side, P, T, H, k, keep_idx, scale,
                                                              zero, static_cast<OutT*>(out), ldo, S, chunks, rpc);
  return launched();
}

template <typename OutT>
hq_status launch_fused(const uint16_t* x, int ldx, int P, int T, int H, int k, const int32_t* keep_idx,
                       const float* scale, const float* inv_scale, const uint8_t* zero, void* out, int ldo,
                       cudaStream_t st, DeviceInfo& d) {
  const int S = (H + hq::kFuSlice - 1) / hq::kFuSlice;
  CUtensorMap map;
  if (!encode_2d(&map, x, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)H, (uint64_t)P * T, hq::kFuSlice,
                 hq::kFuTileRows, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, (uint64_t)ldx * 2))
    return HQ_ERR_CUDA;
  const size_t smem = hq::fu_smem_bytes(P);
  auto kern = hq::compress_reduce_kernel<OutT>;
  int per_sm = 0;
  if (occupancy(d.fused[std::is_same<OutT, float>::value ? 1 : 0], kern, hq::kFuThreads, smem, P, &per_sm) != HQ_OK)
    return HQ_ERR_CUDA;
  // one wave that fills every resident CTA slot (wave_chunks)
  const WaveChunks wc = wave_chunks((long long)d.sms * per_sm, S, (T + hq::kFuTileRows - 1) / hq::kFuTileRows);
  kern<<<(unsigned)(S * wc.base + wc.extra), hq::kFuThreads, smem, st>>>(map, P, T, H, k, keep_idx, scale, inv_scale,
                                                                          zero, static_cast<OutT*>(out), ldo, S,
                                                                          wc.base, wc.extra, wait_limits());
  return launched();
}

// hq_read_device_error: the error word is taken and cleared in one atomic exchange, so an error a
// kernel on another stream records at the same moment lands either in this read or in the word
// for the next one; the value goes through a second device word to the host.
__device__ unsigned int g_error_taken = 0;
__global__ void take_error_kernel() { g_error_taken = atomicExch(&hq::g_error_word, 0u); }
std::mutex g_error_mu;  // one read at a time per process (they share g_error_taken)

// Bounded-wait self-test: one thread waits on an mbarrier that nothing arrives on.
__global__ void selftest_wait_kernel(long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  hq::mbar_init(&bar, 1);
  abort = 0;
  hq::fence_barrier_init();
  hq::mbar_wait(&bar, 0, &abort, limit);
}

// A leading dimension: at least the width, and rows of a multiple of 16 bytes.
bool ld_ok(int ld, int H) { return ld >= H && ld % 8 == 0; }

// Argument checks and launch shared by the two reductions (kShard: each rank's value rounded to
// bf16 before it is added); the output has a row pitch of ldo elements.
template <bool kShard>
hq_status dequant_entry(const uint32_t* codes, const uint16_t* side, int P, int T, int H, int k,
                        const int32_t* keep_idx, const int32_t* rest_idx, const float* scale,
                        const uint8_t* zero, void* out, int ldo, hq_out_dtype out_dtype, void* stream) {
  if (check_shape(P, H, k) != HQ_OK || T < 0 || !ld_ok(ldo, H)) return HQ_ERR_INVALID_ARG;
  if (out_dtype != HQ_OUT_BF16 && out_dtype != HQ_OUT_F32) return HQ_ERR_INVALID_ARG;
  if (!scale || !zero) return HQ_ERR_INVALID_ARG;
  if ((k > 0 && !keep_idx) || (k < H && !rest_idx)) return HQ_ERR_INVALID_ARG;
  if (T > 0 && (!out || (k > 0 && !side) || (k < H && !codes))) return HQ_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(side, 16) || !aligned(codes, 4) || !aligned(scale, 16) ||
      !aligned(zero, 16) || !aligned(keep_idx, 4) || !aligned(rest_idx, 4))
    return HQ_ERR_MISALIGNED;
  if (T == 0) return HQ_OK;
  DeviceInfo* d = nullptr;
  if (device_info(&d) != HQ_OK) return HQ_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  WireSrc src;
  src.codes = codes;
  src.side = side;
  if (out_dtype == HQ_OUT_BF16)
    return launch_dequant<uint16_t, kShard>(src, P, T, H, k, keep_idx, scale, zero, out, ldo, st, *d);
  return launch_dequant<float, kShard>(src, P, T, H, k, keep_idx, scale, zero, out, ldo, st, *d);
}

// The wires of the P ranks in P separate buffers (each possibly a peer GPU's memory).
hq_status dequant_ranks_entry(const uint32_t* const* codes, const uint16_t* const* side, int P, int T, int H, int k,
                              const int32_t* keep_idx, const int32_t* rest_idx, const float* scale,
                              const uint8_t* zero, void* out, hq_out_dtype out_dtype, void* stream) {
  if (check_shape(P, H, k) != HQ_OK || P > hq::kMaxRankMaps || T < 0) return HQ_ERR_INVALID_ARG;
  if (H - k < 32 || (H - k) % 32 != 0) return HQ_ERR_INVALID_ARG;  // code rows staged by TMA
  if (out_dtype != HQ_OUT_BF16 && out_dtype != HQ_OUT_F32) return HQ_ERR_INVALID_ARG;
  if (!scale || !zero || !rest_idx || (k > 0 && !keep_idx)) return HQ_ERR_INVALID_ARG;
  if (T > 0) {
    if (!out || !codes || (k > 0 && !side)) return HQ_ERR_INVALID_ARG;
    for (int r = 0; r < P; ++r) {
      if (!codes[r] || (k > 0 && !side[r])) return HQ_ERR_INVALID_ARG;
      if (!aligned(codes[r], 16) || (k > 0 && !aligned(side[r], 16))) return HQ_ERR_MISALIGNED;
    }
  }
  if (!aligned(out, 16) || !aligned(scale, 16) || !aligned(zero, 16) || !aligned(keep_idx, 4) ||
      !aligned(rest_idx, 4))
    return HQ_ERR_MISALIGNED;
  if (T == 0) return HQ_OK;
  DeviceInfo* d = nullptr;
  if (device_info(&d) != HQ_OK) return HQ_ERR_CUDA;
  WireSrc src;
  src.codes_r = codes;
  src.side_r = k > 0 ? side : nullptr;
  src.per_rank = true;
  if (k == 0) {
    static const uint16_t* const kNone[hq::kMaxRankMaps] = {};
    src.side_r = kNone;
  }
  cudaStream_t st = (cudaStream_t)stream;
  if (out_dtype == HQ_OUT_BF16)
    return launch_dequant<uint16_t, false>(src, P, T, H, k, keep_idx, scale, zero, out, H, st, *d);
  return launch_dequant<float, false>(src, P, T, H, k, keep_idx, scale, zero, out, H, st, *d);
}

hq_status calibrate_entry(const uint16_t* x, int ldx, int P, int T, int H, float beta, int first_batch,
                          float* ema_min, float* ema_max, void* stream) {
  if (check_shape(P, H, 0) != HQ_OK || T < 1 || !ld_ok(ldx, H)) return HQ_ERR_INVALID_ARG;
  if (!(beta >= 0.0f && beta < 1.0f)) return HQ_ERR_INVALID_ARG;
  if (!x || !ema_min || !ema_max) return HQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(ema_min, 16) || !aligned(ema_max, 16)) return HQ_ERR_MISALIGNED;
  const float one_minus_beta = 1.0f - beta;
  dim3 grid((unsigned)((H + hq::kCalCols - 1) / hq::kCalCols), (unsigned)P);
  hq::calibrate_kernel<<<grid, hq::kCalThreads, 0, (cudaStream_t)stream>>>(
      x, ldx, T, H, beta, one_minus_beta, first_batch ? 1 : 0, ema_min, ema_max);
  return launched();
}

hq_status quantize_entry(const uint16_t* x, int ldx, int P, int T, int H, int k, const int32_t* keep_idx,
                         const int32_t* rest_idx, const float* inv_scale, const uint8_t* zero, uint32_t* codes,
                         uint16_t* side, void* stream) {
  if (check_shape(P, H, k) != HQ_OK || T < 0 || !ld_ok(ldx, H)) return HQ_ERR_INVALID_ARG;
  if (!inv_scale || !zero) return HQ_ERR_INVALID_ARG;
  if ((k > 0 && !keep_idx) || (k < H && !rest_idx)) return HQ_ERR_INVALID_ARG;
  if (T > 0 && (!x || (k > 0 && !side) || (k < H && !codes))) return HQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(side, 16) || !aligned(codes, 4) || !aligned(inv_scale, 16) ||
      !aligned(zero, 16) || !aligned(keep_idx, 4) || !aligned(rest_idx, 4))
    return HQ_ERR_MISALIGNED;
  if (T == 0) return HQ_OK;
  DeviceInfo* d = nullptr;
  if (device_info(&d) != HQ_OK) return HQ_ERR_CUDA;
  const int S = (H + hq::kQtSlice - 1) / hq::kQtSlice;
  CUtensorMap map_x;  // x as 32-bit pairs of bf16: the box is 132 pairs = 264 features wide
  if (!encode_2d(&map_x, x, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)H / 2, (uint64_t)P * T, hq::kQtBoxU32,
                 hq::kQtTileRows, CU_TENSOR_MAP_L2_PROMOTION_NONE,  // 528-byte rows: no 256-byte over-fetch
                 (uint64_t)ldx * 2))
    return HQ_ERR_CUDA;
  // J CTAs per slice, one wave; each takes a balanced contiguous range of (rank, 64-row block) units
  const long long units = (long long)P * ceil_div(T, hq::kQtTileRows);
  long long J = (long long)d->sms * d->qt_blocks / S;
  if (J < 1) J = 1;
  if (J > units) J = units;
  hq::quantize_pack_tma_kernel<<<(unsigned)(S * J), hq::kQtThreads, sizeof(hq::QtSmem) + 128,
                                 (cudaStream_t)stream>>>(map_x, x, ldx, P, T, H, k, keep_idx, rest_idx,
                                                         inv_scale, zero, codes, side, S, (int)J,
                                                         wait_limits());
  return launched();
}

hq_status compress_entry(const uint16_t* x, int ldx, int P, int T, int H, int k, const int32_t* keep_idx,
                         const int32_t* rest_idx, const float* scale, const float* inv_scale, const uint8_t* zero,
                         void* out, int ldo, hq_out_dtype out_dtype, uint32_t* codes_or_null,
                         uint16_t* side_or_null, void* stream) {
  if (check_shape(P, H, k) != HQ_OK || T < 0 || !ld_ok(ldx, H) || !ld_ok(ldo, H)) return HQ_ERR_INVALID_ARG;
  if (out_dtype != HQ_OUT_BF16 && out_dtype != HQ_OUT_F32) return HQ_ERR_INVALID_ARG;
  if (!scale || !inv_scale || !zero) return HQ_ERR_INVALID_ARG;
  if ((k > 0 && !keep_idx) || (k < H && !rest_idx)) return HQ_ERR_INVALID_ARG;
  if (T > 0 && (!x || !out)) return HQ_ERR_INVALID_ARG;
  const bool wire = codes_or_null || side_or_null;
  if (T > 0 && wire && ((k > 0 && !side_or_null) || (k < H && !codes_or_null))) return HQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16) || !aligned(scale, 16) || !aligned(inv_scale, 16) ||
      !aligned(zero, 16) || !aligned(keep_idx, 4) || !aligned(rest_idx, 4) ||
      !aligned(codes_or_null, 4) || !aligned(side_or_null, 16))
    return HQ_ERR_MISALIGNED;
  if (T == 0) return HQ_OK;
  DeviceInfo* d = nullptr;
  if (device_info(&d) != HQ_OK) return HQ_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  if (wire) {
    const hq_status q = quantize_entry(x, ldx, P, T, H, k, keep_idx, rest_idx, inv_scale, zero, codes_or_null,
                                       side_or_null, stream);
    if (q != HQ_OK) return q;
  }
  if (out_dtype == HQ_OUT_BF16)
    return launch_fused<uint16_t>(x, ldx, P, T, H, k, keep_idx, scale, inv_scale, zero, out, ldo, st, *d);
  return launch_fused<float>(x, ldx, P, T, H, k, keep_idx, scale, inv_scale, zero, out, ldo, st, *d);
}

// The two-step all-reduce's workspace: step-1 wire (codes, side), the reduced tensor, and the P
// reducers' step-2 wires, each region 256-byte aligned.
struct TwoStepLayout {
  size_t codes, side, red, codes2, side2, total;
};
size_t round256(size_t n) { return (n + 255) & ~size_t(255); }
TwoStepLayout two_step_layout(int P, int T, int H, int k, int k2) {
  TwoStepLayout L;
  size_t off = 0;
  L.codes = off;
  off += round256((size_t)P * T * (H - k) / 2);
  L.side = off;
  off += round256((size_t)P * k * T * 2);
  L.red = off;
  off += round256((size_t)T * H * 2);
  L.codes2 = off;
  off += round256((size_t)T * (H - k2) / 2);  // P blocks of T/P rows
  L.side2 = off;
  off += round256((size_t)k2 * T * 2);
  L.total = off;
  return L;
}

hq_status two_step_entry(const uint16_t* x, int P, int T, int H, int k, const int32_t* keep_idx,
                         const int32_t* rest_idx, const float* scale, const float* inv_scale, const uint8_t* zero,
                         int k2, const int32_t* keep2, const int32_t* rest2, const float* scale2,
                         const float* inv_scale2, const uint8_t* zero2, void* workspace, size_t workspace_bytes,
                         void* out, hq_out_dtype out_dtype, void* stream) {
  if (check_shape(P, H, k) != HQ_OK || check_shape(P, H, k2) != HQ_OK || T < 0 || T % P != 0 || H % 16 != 0)
    return HQ_ERR_INVALID_ARG;  // H % 16: every reducer's row of zero2 starts on a 16-byte boundary
  if (out_dtype != HQ_OUT_BF16 && out_dtype != HQ_OUT_F32) return HQ_ERR_INVALID_ARG;
  if (!scale2 || !inv_scale2 || !zero2 || (k2 > 0 && !keep2) || (k2 < H && !rest2)) return HQ_ERR_INVALID_ARG;
  if (T > 0 && !out) return HQ_ERR_INVALID_ARG;
  if (!aligned(scale2, 16) || !aligned(inv_scale2, 16) || !aligned(zero2, 16) || !aligned(keep2, 4) ||
      !aligned(rest2, 4) || !aligned(out, 16))
    return HQ_ERR_MISALIGNED;
  if (T == 0) return HQ_OK;
  const TwoStepLayout L = two_step_layout(P, T, H, k, k2);
  if (!workspace || workspace_bytes < L.total) return HQ_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return HQ_ERR_MISALIGNED;
  char* ws = static_cast<char*>(workspace);
  uint32_t* codes = reinterpret_cast<uint32_t*>(ws + L.codes);
  uint16_t* side = reinterpret_cast<uint16_t*>(ws + L.side);
  uint16_t* red = reinterpret_cast<uint16_t*>(ws + L.red);
  uint32_t* codes2 = reinterpret_cast<uint32_t*>(ws + L.codes2);
  uint16_t* side2 = reinterpret_cast<uint16_t*>(ws + L.side2);
  // step 1: every rank's wire, the rank-ordered reduction into the reduced tensor (bf16)
  hq_status st = quantize_entry(x, H, P, T, H, k, keep_idx, rest_idx, inv_scale, zero, codes, side, stream);
  if (st != HQ_OK) return st;
  st = dequant_entry<false>(codes, side, P, T, H, k, keep_idx, rest_idx, scale, zero, red, H, HQ_OUT_BF16, stream);
  if (st != HQ_OK) return st;
  // step 2: reducer j re-quantizes its row block with grid row j, and the block is dequantized
  // with it.  The reduced tensor [T][H] is [P][T/P][H]: reducer j's block is "rank" j of one
  // quantize-pack call (whose output layout is exactly the P step-2 wires, block after block),
  // and the P blocks are P independent one-rank problems of one batched dequant-reduce launch.
  const int Tb = T / P;
  st = quantize_entry(red, H, P, Tb, H, k2, keep2, rest2, inv_scale2, zero2, codes2, side2, stream);
  if (st != HQ_OK) return st;
  if (Tb == 0) return HQ_OK;
  DeviceInfo* d = nullptr;
  if (device_info(&d) != HQ_OK) return HQ_ERR_CUDA;
  WireSrc src;
  src.codes = codes2;
  src.side = side2;
  if (out_dtype == HQ_OUT_BF16)
    return launch_dequant<uint16_t, false>(src, 1, Tb, H, k2, keep2, scale2, zero2, out, H, (cudaStream_t)stream, *d, P);
  return launch_dequant<float, false>(src, 1, Tb, H, k2, keep2, scale2, zero2, out, H, (cudaStream_t)stream, *d, P);
}

// Scratch of hq_two_step_reduce_noalloc: a fixed array in every device's global memory, so that a
// caller that may not allocate device memory needs no workspace.  In host code the array's name
// only stands for it; its device address is fetched once per device (device_scratch) and passed to
// the kernels like any workspace pointer.
constexpr size_t kNoAllocScratchBytes = HQ_TWO_STEP_NOALLOC_MAX_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// The current device's address of g_noalloc_scratch, looked up on the first call on that device.
hq_status device_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return HQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HQ_OK;
}

}  // namespace

extern "C" {

hq_status hq_two_step_reduce_noalloc(const uint16_t* x, int P, int T, int H, int k, const int32_t* keep_idx,
                                     const int32_t* rest_idx, const float* scale, const float* inv_scale,
                                     const uint8_t* zero, int k2, const int32_t* keep2, const int32_t* rest2,
                                     const float* scale2, const float* inv_scale2, const uint8_t* zero2, void* out,
                                     hq_out_dtype out_dtype, void* stream) {
  const size_t need = hq_two_step_workspace_bytes(P, T, H, k, k2);
  if (need == 0 || need > kNoAllocScratchBytes) return HQ_ERR_INVALID_ARG;  // rejected before any launch
  void* scratch = nullptr;
  if (device_scratch(&scratch) != HQ_OK) return HQ_ERR_CUDA;
  return two_step_entry(x, P, T, H, k, keep_idx, rest_idx, scale, inv_scale, zero, k2, keep2, rest2, scale2,
                        inv_scale2, zero2, scratch, kNoAllocScratchBytes, out, out_dtype, stream);
}

size_t hq_two_step_workspace_bytes(int P, int T, int H, int k, int k2) {
  if (check_shape(P, H, k) != HQ_OK || check_shape(P, H, k2) != HQ_OK || T < 0) return 0;
  return two_step_layout(P, T, H, k, k2).total;
}

hq_status hq_two_step_reduce(const uint16_t* x, int P, int T, int H, int k, const int32_t* keep_idx,
                             const int32_t* rest_idx, const float* scale, const float* inv_scale, const uint8_t* zero,
                             int k2, const int32_t* keep2, const int32_t* rest2, const float* scale2,
                             const float* inv_scale2, const uint8_t* zero2, void* workspace, size_t workspace_bytes,
                             void* out, hq_out_dtype out_dtype, void* stream) {
  return two_step_entry(x, P, T, H, k, keep_idx, rest_idx, scale, inv_scale, zero, k2, keep2, rest2, scale2,
                        inv_scale2, zero2, workspace, workspace_bytes, out, out_dtype, stream);
}

hq_status hq_calibrate(const uint16_t* x, int P, int T, int H, float beta, int first_batch,
                       float* ema_min, float* ema_max, void* stream) {
  return calibrate_entry(x, H, P, T, H, beta, first_batch, ema_min, ema_max, stream);
}

hq_status hq_calibrate_ld(const uint16_t* x, int ldx, int P, int T, int H, float beta, int first_batch,
                          float* ema_min, float* ema_max, void* stream) {
  return calibrate_entry(x, ldx, P, T, H, beta, first_batch, ema_min, ema_max, stream);
}

hq_status hq_select_topk(const float* ema_min, const float* ema_max, int P, int H, int k,
                         int32_t* keep_idx, int32_t* rest_idx, float* scale, float* inv_scale,
                         uint8_t* zero, void* stream) {
  if (check_shape(P, H, k) != HQ_OK) return HQ_ERR_INVALID_ARG;
  if (!ema_min || !ema_max || !scale || !inv_scale || !zero) return HQ_ERR_INVALID_ARG;
  if ((k > 0 && !keep_idx) || (k < H && !rest_idx)) return HQ_ERR_INVALID_ARG;
  if (!aligned(ema_min, 16) || !aligned(ema_max, 16) || !aligned(scale, 16) ||
      !aligned(inv_scale, 16) || !aligned(zero, 16) || !aligned(keep_idx, 4) || !aligned(rest_idx, 4))
    return HQ_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (device_info(&d) != HQ_OK) return HQ_ERR_CUDA;
  const size_t smem = (size_t)H * sizeof(uint32_t);
  {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (!d->select_smem_set) {
      if (cudaFuncSetAttribute(hq::select_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(hq::kMaxH * sizeof(uint32_t))) != cudaSuccess)
        return HQ_ERR_CUDA;
      d->select_smem_set = true;
    }
  }
  // parameters and keys over the whole GPU, then the selection in one CTA (same stream)
  const unsigned pgrid = (unsigned)ceil_div(H, hq::kSelParamFeatures);
  hq::select_params_kernel<<<pgrid, hq::kSelParamThreads, 0, (cudaStream_t)stream>>>(
      ema_min, ema_max, P, H, k, keep_idx, rest_idx, scale, inv_scale, zero);
  if (cudaGetLastError() != cudaSuccess) return HQ_ERR_CUDA;
  hq::select_topk_kernel<<<1, hq::kSelThreads, smem, (cudaStream_t)stream>>>(H, k, keep_idx, rest_idx);
  return launched();
}

hq_status hq_quantize_pack(const uint16_t* x, int P, int T, int H, int k, const int32_t* keep_idx,
                           const int32_t* rest_idx, const float* inv_scale, const uint8_t* zero,
                           uint32_t* codes, uint16_t* side, void* stream) {
  return quantize_entry(x, H, P, T, H, k, keep_idx, rest_idx, inv_scale, zero, codes, side, stream);
}

hq_status hq_quantize_pack_ld(const uint16_t* x, int ldx, int P, int T, int H, int k, const int32_t* keep_idx,
                              const int32_t* rest_idx, const float* inv_scale, const uint8_t* zero,
                              uint32_t* codes, uint16_t* side, void* stream) {
  return quantize_entry(x, ldx, P, T, H, k, keep_idx, rest_idx, inv_scale, zero, codes, side, stream);
}

hq_status hq_dequant_reduce(const uint32_t* codes, const uint16_t* side, int P, int T, int H, int k,
                            const int32_t* keep_idx, const int32_t* rest_idx, const float* scale,
                            const uint8_t* zero, void* out, hq_out_dtype out_dtype, void* stream) {
  return dequant_entry<false>(codes, side, P, T, H, k, keep_idx, rest_idx, scale, zero, out, H, out_dtype, stream);
}

hq_status hq_dequant_reduce_ld(const uint32_t* codes, const uint16_t* side, int P, int T, int H, int k,
                               const int32_t* keep_idx, const int32_t* rest_idx, const float* scale,
                               const uint8_t* zero, void* out, int ldo, hq_out_dtype out_dtype, void* stream) {
  return dequant_entry<false>(codes, side, P, T, H, k, keep_idx, rest_idx, scale, zero, out, ldo, out_dtype,
                              stream);
}

hq_status hq_dequant_reduce_ranks(const uint32_t* const* codes, const uint16_t* const* side, int P, int T, int H,
                                  int k, const int32_t* keep_idx, const int32_t* rest_idx, const float* scale,
                                  const uint8_t* zero, void* out, hq_out_dtype out_dtype, void* stream) {
  return dequant_ranks_entry(codes, side, P, T, H, k, keep_idx, rest_idx, scale, zero, out, out_dtype, stream);
}

hq_status hq_dequant_reduce_bf16_shards(const uint32_t* codes, const uint16_t* side, int P, int T, int H, int k,
                                        const int32_t* keep_idx, const int32_t* rest_idx, const float* scale,
                                        const uint8_t* zero, void* out, hq_out_dtype out_dtype, void* stream) {
  return dequant_entry<true>(codes, side, P, T, H, k, keep_idx, rest_idx, scale, zero, out, H, out_dtype, stream);
}

hq_status hq_compress_reduce(const uint16_t* x, int P, int T, int H, int k, const int32_t* keep_idx,
                             const int32_t* rest_idx, const float* scale, const float* inv_scale,
                             const uint8_t* zero, void* out, hq_out_dtype out_dtype,
                             uint32_t* codes_or_null, uint16_t* side_or_null, void* stream) {
  return compress_entry(x, H, P, T, H, k, keep_idx, rest_idx, scale, inv_scale, zero, out, H, out_dtype,
                        codes_or_null, side_or_null, stream);
}

hq_status hq_compress_reduce_ld(const uint16_t* x, int ldx, int P, int T, int H, int k, const int32_t* keep_idx,
                                const int32_t* rest_idx, const float* scale, const float* inv_scale,
                                const uint8_t* zero, void* out, int ldo, hq_out_dtype out_dtype,
                                uint32_t* codes_or_null, uint16_t* side_or_null, void* stream) {
  return compress_entry(x, ldx, P, T, H, k, keep_idx, rest_idx, scale, inv_scale, zero, out, ldo, out_dtype,
                        codes_or_null, side_or_null, stream);
}

const char* hq_status_string(hq_status s) {
  switch (s) {
    case HQ_OK: return "HQ_OK";
    case HQ_ERR_INVALID_ARG: return "HQ_ERR_INVALID_ARG";
    case HQ_ERR_MISALIGNED: return "HQ_ERR_MISALIGNED";
    case HQ_ERR_CUDA: return "HQ_ERR_CUDA";
    case HQ_ERR_TIMEOUT: return "HQ_ERR_TIMEOUT";
    case HQ_ERR_BAD_INDEX: return "HQ_ERR_BAD_INDEX";
  }
  return "HQ_ERR_UNKNOWN";
}

hq_status hq_read_device_error(void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  std::lock_guard<std::mutex> lock(g_error_mu);
  take_error_kernel<<<1, 1, 0, st>>>();
  if (cudaGetLastError() != cudaSuccess) return HQ_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_error_taken, sizeof v, 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return HQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return HQ_ERR_CUDA;
  return (hq_status)v;
}

hq_status hq_selftest_bounded_wait(long long limit_cycles, void* stream) {
  if (limit_cycles < 0) return HQ_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(limit_cycles);
  return launched();
}

hq_status hq_selftest_set_pipeline_stall(long long consumer_limit_cycles, long long producer_delay_cycles) {
  if (consumer_limit_cycles < 0 || producer_delay_cycles < 0 || producer_delay_cycles > kMaxStallDelayCycles)
    return HQ_ERR_INVALID_ARG;
  if ((consumer_limit_cycles == 0) != (producer_delay_cycles == 0)) return HQ_ERR_INVALID_ARG;
  g_stall_consumer_limit.store(consumer_limit_cycles);
  g_stall_producer_delay.store(producer_delay_cycles);
  return HQ_OK;
}

int64_t hq_wire_bytes_per_row(int H, int k) {
  if (H < 0 || k < 0 || k > H) return -1;
  return (int64_t)(H - k) / 2 + 2 * (int64_t)k;
}

}  // extern "C"
