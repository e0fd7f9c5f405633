// Host-only checks of the launch-shape helpers (no GPU call is made):
// layout::split_tokens (blocks and chunk of a layout launch) and row_slices
// (column slices of the copy kernels).  Prints "ok" or the first failure.
#include <cstdio>

#include "layout_common.cuh"

using moe::layout::split_tokens;
using moe::layout::kMaxBlocks;

static int fail(const char *what, long a, long b, long c) {
  std::printf("FAIL %s (%ld, %ld, %ld)\n", what, a, b, c);
  return 1;
}

int main() {
  const int Ts[] = {1, 7, 8, 31, 32, 33, 255, 256, 257, 1000, 8192, 32768, 65536, 100000, 140000, 1 << 20};
  const int maxes[] = {1, 2, 8, 148, 296, 512, 592, 4096};
  for (int T : Ts)
    for (int mb : maxes)
      for (int g : {8, 32}) {
        int nblk = 0, chunk = 0;
        split_tokens(T, mb, nblk, chunk, g);
        if (chunk % g != 0 || chunk < g) return fail("chunk not a positive multiple of the granule", T, mb, g);
        if ((long)nblk * chunk < T || (long)(nblk - 1) * chunk >= T)
          return fail("chunks do not cover the tokens exactly", T, mb, g);
        if (nblk > mb && mb >= 1 && mb <= kMaxBlocks) return fail("more blocks than allowed", T, mb, nblk);
        if (nblk > kMaxBlocks) return fail("more blocks than the count table holds", T, mb, nblk);
        // the workspace holds a count-table row per 8 tokens, up to kMaxBlocks
        const long rows = ((long)T + 7) / 8 < kMaxBlocks ? ((long)T + 7) / 8 : kMaxBlocks;
        if (nblk > rows) return fail("more blocks than workspace rows", T, mb, nblk);
      }
  const long rows_[] = {1, 3, 64, 256, 1024, 4096, 8192, 65536, 1 << 20};
  const int nvecs[] = {1, 16, 31, 32, 33, 512, 896, 4096};
  for (long rows : rows_)
    for (int nvec : nvecs)
      for (int sms : {1, 148})
      for (int wps : {16, 32}) {
        int slices = 0, svec = 0;
        moe::row_slices(rows, nvec, sms, slices, svec, wps);
        if (slices < 1 || svec < 1) return fail("empty slicing", rows, nvec, sms);
        if ((long)slices * svec < nvec || (long)(slices - 1) * svec >= nvec)
          return fail("slices do not cover the row exactly", rows, nvec, slices);
        if (slices > 1 && svec % 32 != 0) return fail("a slice is not whole warp-widths", rows, nvec, svec);
        if (rows >= (long)wps * sms && slices != 1) return fail("many rows should keep one slice", rows, nvec, slices);
        if ((long)rows * slices >= (1L << 31)) return fail("work items overflow 31 bits", rows, nvec, slices);
      }
  std::printf("ok\n");
  return 0;
}
