// Host-side check of the work-splitting arithmetic the kernels share (built and
// run by tests/test_host_plan.py; no GPU needed): equal pieces of a flattened
// stream, the owner of each unit, the automatic piece count, and the units of a
// segment (its tiles plus the empty units standing for its fixed cost).
#include <cstdio>
#include <cstdlib>

#include "pa_device.cuh"

static int fails = 0;
#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      if (++fails < 20) std::printf("FAIL line %d: %s\n", __LINE__, #c); \
    }                                                              \
  } while (0)

int main() {
  unsigned long long rng = 12345;
  auto next = [&]() {
    rng = rng * 6364136223846793005ull + 1442695040888963407ull;
    return rng >> 33;
  };
  for (int iter = 0; iter < 20000; ++iter) {
    const long long total = 1 + static_cast<long long>(next() % (iter < 10000 ? 5000 : 50000000));
    const int parts = 1 + static_cast<int>(next() % 20000);
    // pieces tile [0, total) in order, with sizes differing by at most one
    CHECK(pa::piece_begin(0, total, parts) == 0);
    CHECK(pa::piece_begin(parts, total, parts) == total);
    long long lo = total, hi = 0;
    for (int k = 0; k < 64; ++k) {
      const long long c = static_cast<long long>(next() % parts);
      const long long b0 = pa::piece_begin(c, total, parts), b1 = pa::piece_begin(c + 1, total, parts);
      CHECK(b0 <= b1);
      lo = b1 - b0 < lo ? b1 - b0 : lo;
      hi = b1 - b0 > hi ? b1 - b0 : hi;
    }
    CHECK(hi - lo <= 1);
    // the owner of unit t is the piece whose range holds it
    for (int k = 0; k < 64; ++k) {
      const long long t = static_cast<long long>(next() % total);
      const int o = pa::piece_of(t, total, parts);
      CHECK(o >= 0 && o < parts);
      CHECK(pa::piece_begin(o, total, parts) <= t && t < pa::piece_begin(o + 1, total, parts));
    }
    // automatic counts: within [1, parts]; between the floor and the launch size
    // the count is the fewest pieces of at most min_units units each; an explicit
    // count (min_units 0) is kept
    const int min_units = static_cast<int>(next() % 17);
    const long long floor_pieces = 1 + static_cast<long long>(next() % 2048);
    const int used = pa::used_pieces(parts, total, min_units, floor_pieces);
    CHECK(used >= 1 && used <= parts);
    if (min_units == 0) {
      CHECK(used == parts);
    } else if (used < parts && used > floor_pieces) {
      CHECK(static_cast<long long>(used) * min_units >= total);          // pieces <= min_units
      CHECK(static_cast<long long>(used - 1) * min_units < total);       // and no fewer would do
    } else if (used < parts) {
      CHECK(used == floor_pieces);                                       // the floor holds
    }
  }
  // units of a sequence: tiles plus extra, none for an empty one; clamped to cap
  CHECK(pa::seq_units(0, 1000, 16, 2) == 0);
  CHECK(pa::seq_units(1, 1000, 16, 2) == 3);
  CHECK(pa::seq_units(16, 1000, 16, 2) == 3);
  CHECK(pa::seq_units(17, 1000, 16, 2) == 4);
  CHECK(pa::seq_units(5000, 1000, 16, 0) == 63);
  CHECK(pa::seq_units(-7, 1000, 16, 2) == 0);
  std::printf(fails ? "host plan check: %d failures\n" : "host plan check: ok\n", fails);
  return fails ? 1 : 0;
}
