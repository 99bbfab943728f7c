/*
 * hq_synth_gpu.cu -- device side of the synthetic partial-sum generator.
 *
 * Fills a whole batch x[P][T][H] (bf16 bits) on the GPU with exactly the values the
 * host generator (hq_synth.c) produces: both compile the same hq_synth_core.h, this
 * file with -fmad=false so that no multiply-add is contracted.  Full-size inputs
 * (up to several GiB per batch) are made here in milliseconds instead of minutes.
 *
 * Holds none of the compression method's arithmetic.
 */
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "hq_synth_core.h"

namespace {

constexpr int kMaxRanks = 64;

struct RankKeys {
  uint64_t k[kMaxRanks];
};

__global__ void syn_fill_kernel(RankKeys keys, int P, int T, int H, int dist,
                                const double* __restrict__ colscale, double spike_p,
                                double spike_mult, uint16_t* __restrict__ out) {
  const uint64_t per_rank = (uint64_t)T * (uint64_t)H;
  const uint64_t total = per_rank * (uint64_t)P;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int r = (int)(i / per_rank);
    const uint64_t elem = i - (uint64_t)r * per_rank; /* t*H + h */
    const int h = (int)(elem % (uint64_t)H);
    const double cs = colscale ? colscale[h] : 1.0;
    out[i] = syn_element(keys.k[r], elem, dist, cs, spike_p, spike_mult);
  }
}

}  // namespace

extern "C" int syn_fill_gpu(uint64_t seed, int purpose, int batch, int P, int T, int H, int dist,
                            const double* colscale_dev, double spike_p, double spike_mult,
                            uint16_t* out_dev, void* stream) {
  if (P < 1 || P > kMaxRanks || T < 1 || H < 1 || out_dev == nullptr) return 1;
  RankKeys keys;
  for (int r = 0; r < P; ++r) keys.k[r] = syn_key(seed, (uint64_t)purpose, (uint64_t)batch, (uint64_t)r);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const uint64_t total = (uint64_t)P * (uint64_t)T * (uint64_t)H;
  uint64_t blocks = (total + 255) / 256;
  const uint64_t cap = (uint64_t)sms * 16;
  if (blocks > cap) blocks = cap;
  syn_fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      keys, P, T, H, dist, colscale_dev, spike_p, spike_mult, out_dev);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
