// Bit packing of low-bit codes (gptq-for-llama article, ainews.cool, "工程细节": four
// 4-bit codes per 16-bit integer).  One thread per output word: word w of a row
// holds bits [32w, 32w + 32) of the row's LSB-first stream of `bits`-bit fields,
// so consecutive threads read consecutive codes and write consecutive words.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace gptq {

__global__ void k_pack(const uint8_t* __restrict__ codes, int64_t R, int64_t C, int bits,
                       int64_t nw, uint32_t* __restrict__ packed) {
  const int64_t total = R * nw;
  const uint32_t mask = (1u << bits) - 1u;
  for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = idx / nw, w = idx % nw;
    const int64_t b0 = 32 * w;
    const int64_t c0 = b0 / bits;
    const int64_t c1 = min(C - 1, (b0 + 31) / bits);
    const uint8_t* row = codes + r * C;
    uint64_t acc = 0;
    for (int64_t c = c0; c <= c1; ++c) {
      const int64_t sh = c * bits - b0;
      const uint64_t v = row[c] & mask;
      acc |= sh >= 0 ? (v << sh) : (v >> (-sh));
    }
    packed[idx] = uint32_t(acc & 0xffffffffull);
  }
}

gptq_status pack_run(cudaStream_t st, const uint8_t* codes, int64_t R, int64_t C, int bits,
                     uint32_t* packed) {
  const int64_t nw = (C * bits + 31) / 32;
  const int64_t total = R * nw;
  if (total == 0) return GPTQ_OK;
  const int blocks = int(std::min<int64_t>((total + 255) / 256, 148 * 32));
  GPTQ_LAUNCH(k_pack, blocks, 256, 0, st, codes, R, C, bits, nw, packed);
  return GPTQ_OK;
}

}  // namespace gptq
