// Host-side check of the decode kernel's shared-memory layout helpers
// (row ownership, owner-order slots, 128-byte swizzle positions). Built and run
// by tests/test_layout.py; exit status = number of violations.
#include <cstdio>

#include "gdr_decode_tma.cuh"

template <int DK, int R>
int check() {
  constexpr int RL = DK / R, CL = 32 / RL;
  int bad = 0;
  bool seen_row[256] = {};
  bool seen_slot[512] = {};
  for (int rl = 0; rl < RL; ++rl)
    for (int r = 0; r < R; ++r) {
      const int i = r * RL + gdr::row_perm<RL>(rl);  // row held at (rl, r)
      if (i < 0 || i >= DK || seen_row[i]) ++bad;
      else seen_row[i] = true;
      const int slot = gdr::owner_slot<RL, R>(i);
      if (slot != rl * (R + 4) + r || slot >= DK + 4 * RL || seen_slot[slot]) ++bad;
      else seen_slot[slot] = true;
    }
  // The 8 lanes of each quarter-warp read distinct 16-byte swizzle positions.
  for (int q = 0; q < 4; ++q)
    for (int r = 0; r < R; ++r)
      for (int band = 0; band < 64; band += CL * 8) {
        bool pos[8] = {};
        for (int l = 8 * q; l < 8 * q + 8; ++l) {
          const int rl = l / CL, cg = l % CL;
          const int i = r * RL + gdr::row_perm<RL>(rl);
          const int off = gdr::swz_offset<DK>(i, band + cg * 8);
          const int p = (off >> 4) & 7;
          if (pos[p]) ++bad;
          pos[p] = true;
        }
      }
  // Per-row vectors: the row lanes of a quarter-warp start in different banks.
  for (int q = 0; q < 4; ++q) {
    int first = -1;
    for (int l = 8 * q; l < 8 * q + 8; ++l) {
      const int bank = ((l / CL) * (R + 4) * 16 / 4) % 32;  // float4 entries
      if (l % CL == 0) {
        if (first == bank) ++bad;
        first = bank;
      }
    }
  }
  std::printf("D_k=%d rows/thread=%d: %s\n", DK, R, bad ? "FAIL" : "ok");
  return bad;
}

int main() { return check<64, 8>() + check<64, 16>() + check<128, 8>() + check<128, 16>(); }
