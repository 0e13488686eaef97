// qsa_synth/gen_host.cu -- host-side fill of seeded synthetic inputs (input generation only).
//
// The same counter-based values as gen_device.cu and the numpy twin in qsa_synth/__init__.py,
// computed on the host cores with a few threads, so that the host can regenerate the inputs of a
// million-token context in seconds (the oracle's side of a parity test or of a CPU baseline).
// Rows of `width` consecutive elements start at arbitrary logical indices.
#include <stdint.h>

#include <thread>
#include <vector>

#include "gen_core.h"

extern "C" int qsyn_fill_rows_host(void* out, const int64_t* starts, int64_t nrows, int64_t width,
                                   uint64_t seed, uint64_t tid, int dist, int threads) {
  if (nrows <= 0 || width <= 0) return 0;
  if (!out || !starts) return 1;
  const uint64_t key = qsyn_key(seed, tid);
  uint16_t* o = static_cast<uint16_t*>(out);
  const int64_t total = nrows * width;
  int nt = threads > 0 ? threads : (int)std::thread::hardware_concurrency();
  if (nt < 1) nt = 1;
  if (total < (int64_t)1 << 16) nt = 1;
  if (nt > 64) nt = 64;
  auto work = [&](int k) {
    const int64_t r0 = nrows * k / nt, r1 = nrows * (k + 1) / nt;
    for (int64_t r = r0; r < r1; ++r) {
      const uint64_t s = (uint64_t)starts[r];
      uint16_t* dst = o + r * width;
      for (int64_t e = 0; e < width; ++e) dst[e] = qsyn_value_bf16(qsyn_hash(key, s + (uint64_t)e), dist);
    }
  };
  if (nt == 1) {
    work(0);
    return 0;
  }
  std::vector<std::thread> pool;
  pool.reserve(nt);
  for (int k = 0; k < nt; ++k) pool.emplace_back(work, k);
  for (auto& t : pool) t.join();
  return 0;
}
