// Host check of packed_unit (csrc/attn_internal.h), the work-item mapping of
// the packed-sequence kernels: for many random length mixes, every unit of
// every sequence is reached by exactly one item of the grid row
// 0 .. floor(total / U) + num_seqs - 1, and at most num_seqs items reach none.
// Prints "ok <cases>" or the first failing case; exit status 0 / 1.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../../exact_attention_134_b200/csrc/attn_internal.h"

int main() {
  unsigned long long state = 0x9E3779B97F4A7C15ull;
  auto next = [&]() {  // xorshift64*
    state ^= state >> 12; state ^= state << 25; state ^= state >> 27;
    return (unsigned)((state * 2685821657736338717ull) >> 33);
  };
  const int picks[] = {0, 1, 2, 127, 128, 129, 255, 256, 257, 511, 1000};
  int cases = 0;
  for (int trial = 0; trial < 4000; ++trial) {
    const int n = 1 + (int)(next() % 48);
    const int U = (next() & 1) ? 128 : 256;
    std::vector<int> len(n), off(n + 1, 0);
    for (int s = 0; s < n; ++s) {
      const unsigned r = next() % 12;
      len[s] = r < 11 ? picks[r] : (int)(next() % 3000);
      off[s + 1] = off[s] + len[s];
    }
    const int total = off[n];
    const int items = total / U + n;
    std::vector<int> seen_units(n, 0);
    std::vector<std::vector<char>> hit(n);
    for (int s = 0; s < n; ++s) hit[s].assign((len[s] + U - 1) / U, 0);
    int empty = 0;
    for (int i = 0; i < items; ++i) {
      int rank = -1;
      const int s = attn_sm100::packed_unit(off.data(), n, total, U, i, rank);
      if (s < 0 || s >= n || rank < 0) {
        std::printf("trial %d item %d: sequence %d rank %d out of range\n", trial, i, s, rank);
        return 1;
      }
      if (rank >= (int)hit[s].size()) { ++empty; continue; }
      if (hit[s][rank]) {
        std::printf("trial %d: unit %d of sequence %d reached twice\n", trial, rank, s);
        return 1;
      }
      hit[s][rank] = 1;
    }
    for (int s = 0; s < n; ++s)
      for (size_t u = 0; u < hit[s].size(); ++u)
        if (!hit[s][u]) {
          std::printf("trial %d: unit %zu of sequence %d never reached\n", trial, u, s);
          return 1;
        }
    if (empty > n) {
      std::printf("trial %d: %d empty items for %d sequences\n", trial, empty, n);
      return 1;
    }
    ++cases;
  }
  std::printf("ok %d\n", cases);
  return 0;
}
