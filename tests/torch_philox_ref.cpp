// Library pin for the oracle's Philox4x32-10: PyTorch's own CPU Philox engine
// (ATen/core/PhiloxRNGEngine.h), wrapped in a C function for ctypes.
// The engine's key is (lo32(seed), hi32(seed)) and its counter is
// (lo32(offset), hi32(offset), lo32(subsequence), hi32(subsequence)).
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdint>

extern "C" void torch_philox4x32_10(const uint32_t* ctr, const uint32_t* key, uint32_t* out) {
  uint64_t seed = (uint64_t)key[0] | ((uint64_t)key[1] << 32);
  uint64_t subseq = (uint64_t)ctr[2] | ((uint64_t)ctr[3] << 32);
  uint64_t offset = (uint64_t)ctr[0] | ((uint64_t)ctr[1] << 32);
  at::philox_engine e(seed, 0, 0);
  e.reset_state(seed, subseq);
  e.set_offset(offset);
  for (int i = 0; i < 4; ++i) out[i] = e();
}
