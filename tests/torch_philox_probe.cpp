// Comparator for the Philox4x32-10 pin: runs PyTorch's open-source header-only
// engine (ATen/core/PhiloxRNGEngine.h) on (counter, key) records read from
// stdin and writes the first 128-bit output block of each to stdout.
// The engine's state is key = seed, counter = (offset, subsequence), so a
// counter (c0, c1, c2, c3) is offset c1:c0 and subsequence c3:c2.
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdint>
#include <cstdio>

int main() {
  uint32_t rec[6];
  while (std::fread(rec, sizeof(uint32_t), 6, stdin) == 6) {
    uint64_t seed = (uint64_t(rec[5]) << 32) | rec[4];
    uint64_t subseq = (uint64_t(rec[3]) << 32) | rec[2];
    uint64_t offset = (uint64_t(rec[1]) << 32) | rec[0];
    at::philox_engine eng(seed, subseq, offset);
    uint32_t out[4];
    for (int i = 0; i < 4; ++i) out[i] = eng();
    std::fwrite(out, sizeof(uint32_t), 4, stdout);
  }
  return 0;
}
