// Host-side checks of the kernels' work schedulers (test infrastructure; runs on
// the CPU, no GPU needed).  Includes the kernel headers and calls the same
// __host__ __device__ functions the kernels call:
//  * fwd_decode_tile: every (sequence, head, tile) exactly once; causal tiles
//    longest first inside each group of heads;
//  * fwd_num_kv / fwd256_num_kv: the key-block trip count of a tile equals the
//    blocks its rows' visible keys span (brute force over rows, bottom-right
//    causal alignment, any query / key lengths);
//  * bwd_decode: every (key/value head, key block) exactly once;
//  * decode_splits: splits cover the cache in whole 64-key tiles.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "bwd_kernel.cuh"
#include "decode_kernel.cuh"
#include "fwd256_kernel.cuh"
#include "fwd_kernel.cuh"

using namespace fa;

static int failures = 0;
#define CHECK(cond, ...)                  \
  do {                                    \
    if (!(cond)) {                        \
      if (failures < 20) {                \
        std::printf("FAIL: " __VA_ARGS__); \
        std::printf("\n");                \
      }                                   \
      ++failures;                         \
    }                                     \
  } while (0)

static FwdArgs fwd_args(int B, int H, int Nq, int Nk, int tile_rows, int causal, int hg) {
  FwdArgs a{};
  a.L.B = B;
  a.L.H = H;
  a.L.H_kv = H;
  a.L.Nq = Nq;
  a.L.Nk = Nk;
  a.group = 1;
  a.n_qt = (Nq + tile_rows - 1) / tile_rows;
  a.num_tiles = B * H * a.n_qt;
  a.causal = causal;
  a.heads_per_group = hg;
  return a;
}

static void check_fwd_tiles(int B, int H, int n_rows, int tile_rows, int causal, int hg) {
  const FwdArgs a = fwd_args(B, H, n_rows, n_rows, tile_rows, causal, hg);
  std::vector<int> seen(static_cast<size_t>(a.num_tiles), 0);
  int prev_group = -1, prev_qt = 0;
  for (int t = 0; t < a.num_tiles; ++t) {
    int b, h, qt;
    fwd_decode_tile(a, t, b, h, qt);
    CHECK(b >= 0 && b < B && h >= 0 && h < H && qt >= 0 && qt < a.n_qt, "tile %d out of range", t);
    if (!(b >= 0 && b < B && h >= 0 && h < H && qt >= 0 && qt < a.n_qt)) continue;
    ++seen[(static_cast<size_t>(b) * H + h) * a.n_qt + qt];
    if (causal) {
      const int group = (b * H + h) / hg;
      if (group == prev_group) CHECK(qt <= prev_qt, "causal tiles not longest first (t %d)", t);
      prev_group = group;
      prev_qt = qt;
    }
  }
  for (size_t i = 0; i < seen.size(); ++i) CHECK(seen[i] == 1, "tile %zu visited %d times", i, seen[i]);
}

// brute force: key blocks of `blk` keys that rows [r0, r1) of a sequence see
static int blocks_needed(int nq, int nk, int r0, int r1, int blk, int causal) {
  int need = 0;
  for (int i = r0; i < r1 && i < nq; ++i) {
    const int vis = causal ? (i + nk - nq + 1 < nk ? i + nk - nq + 1 : nk) : nk;
    const int nb = vis <= 0 ? 0 : (vis + blk - 1) / blk;
    if (nb > need) need = nb;
  }
  return need;
}

static void check_num_kv(unsigned seed) {
  std::srand(seed);
  for (int trial = 0; trial < 4000; ++trial) {
    const int nq = std::rand() % 1500, nk = std::rand() % 1500, causal = std::rand() & 1;
    FwdArgs a = fwd_args(1, 1, nq > 0 ? nq : 1, nk, 256, causal, 1);
    SeqSpan s{0, nq, 0, nk, 0};
    for (int qt = 0; qt * 256 < nq + 256; ++qt) {
      const int got = fwd_num_kv(a, s, qt), want = blocks_needed(nq, nk, qt * 256, qt * 256 + 256, 128, causal);
      CHECK(got == want, "fwd_num_kv nq %d nk %d qt %d causal %d: %d != %d", nq, nk, qt, causal, got, want);
    }
    for (int qt = 0; qt * 128 < nq + 128; ++qt) {
      const int got = fwd256_num_kv(a, s, qt), want = blocks_needed(nq, nk, qt * 128, qt * 128 + 128, 64, causal);
      CHECK(got == want, "fwd256_num_kv nq %d nk %d qt %d causal %d: %d != %d", nq, nk, qt, causal, got, want);
    }
  }
}

static void check_bwd_items(int bh_kv, int n_kb, int hg) {
  BwdArgs a{};
  a.bh_kv = bh_kv;
  a.n_kb = n_kb;
  a.heads_per_group = hg;
  std::vector<int> seen(static_cast<size_t>(bh_kv) * n_kb, 0);
  for (int x = 0; x < bh_kv * n_kb; ++x) {
    int bh, kb;
    bwd_decode(a, x, bh, kb);
    const bool in = bh >= 0 && bh < bh_kv && kb >= 0 && kb < n_kb;
    CHECK(in, "bwd item %d out of range", x);
    if (in) ++seen[static_cast<size_t>(bh) * n_kb + kb];
  }
  for (size_t i = 0; i < seen.size(); ++i) CHECK(seen[i] == 1, "bwd item %zu visited %d times", i, seen[i]);
}

static void check_splits() {
  const int bhs[] = {1, 3, 16, 128, 1024, 5000};
  const int nks[] = {1, 63, 64, 65, 1000, 8192, 65536, 1 << 20};
  for (int bh : bhs)
    for (int nk : nks) {
      int sk = 0;
      const int n = decode_splits(bh, nk, &sk);
      CHECK(n >= 1 && sk % 64 == 0 && sk > 0, "splits bh %d nk %d: n %d sk %d", bh, nk, n, sk);
      CHECK(static_cast<long long>(n) * sk >= nk && static_cast<long long>(n - 1) * sk < nk,
            "splits do not cover the cache exactly: bh %d nk %d n %d sk %d", bh, nk, n, sk);
    }
}

int main() {
  const int shapes[][3] = {{1, 1, 128}, {2, 32, 8192}, {1, 16, 65536}, {3, 5, 1000}, {4, 16, 2048}, {1, 7, 257}};
  for (const auto& sh : shapes)
    for (int causal = 0; causal < 2; ++causal)
      for (int tile_rows : {128, 256})
        for (int hg : {1, 3, 12, 48, 1000}) {
          const int bh = sh[0] * sh[1];
          check_fwd_tiles(sh[0], sh[1], sh[2], tile_rows, causal, hg < bh ? hg : bh);
        }
  check_num_kv(12345u);
  for (int bh : {1, 5, 16, 64, 100})
    for (int nkb : {1, 2, 63, 64, 512})
      for (int hg : {1, 2, 5, 9, 1000}) check_bwd_items(bh, nkb, hg < bh ? hg : bh);
  check_splits();
  if (failures) {
    std::printf("%d failures\n", failures);
    return 1;
  }
  std::printf("OK\n");
  return 0;
}
