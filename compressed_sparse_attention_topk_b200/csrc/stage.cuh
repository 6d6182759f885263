// Staging copies: a step's inputs from page-locked host buffers into device
// buffers, and its results back, in one launch.
//
// The pieces are small (tens to a few hundred KB per decode step), so a
// copy-engine transfer costs its fixed latency each time; here every thread
// moves 16-byte pieces through the mapped host buffer itself, so all pieces
// of all copies are in flight at once and the step pays about one round
// trip over the host link.  Host memory is read uncached (ld.global.cv: a
// line the host rewrote since the last launch is fetched again) and written
// through (st.global.wt); device memory takes plain loads and stores.
#pragma once
#include "common.cuh"

namespace csa2 {

constexpr int kStageMax = 16;      // copies per launch
constexpr int kStageThreads = 256;
constexpr int kStageUnroll = 4;    // pieces in flight per thread

struct StageCopy {
  const int4 *src;
  int4 *dst;
  int64_t rows, row16, src16, dst16;  // row length and strides in 16-byte pieces
  int32_t host_src, host_dst;
};

struct StageList {
  StageCopy c[kStageMax];
  int32_t n;
};

// grid = (CTAs per copy, copies).  Piece i of copy y: row i / row16, piece
// i % row16 of that row.
__global__ void __launch_bounds__(kStageThreads) stage_copies_kernel(const StageList L) {
  const StageCopy c = L.c[blockIdx.y];
  const int64_t total = c.rows * c.row16;
  const int64_t step = (int64_t)gridDim.x * kStageThreads;
  for (int64_t base = blockIdx.x * (int64_t)kStageThreads + threadIdx.x; base < total;
       base += step * kStageUnroll) {
    int4 v[kStageUnroll];
    int64_t d[kStageUnroll];
#pragma unroll
    for (int u = 0; u < kStageUnroll; ++u) {
      const int64_t i = base + u * step;
      d[u] = -1;
      if (i < total) {
        const int64_t r = i / c.row16, j = i - r * c.row16;
        const int4 *s = c.src + r * c.src16 + j;
        v[u] = c.host_src ? __ldcv(s) : *s;
        d[u] = r * c.dst16 + j;
      }
    }
#pragma unroll
    for (int u = 0; u < kStageUnroll; ++u) {
      if (d[u] < 0) continue;
      if (c.host_dst)
        __stwt(c.dst + d[u], v[u]);
      else
        c.dst[d[u]] = v[u];
    }
  }
}

}  // namespace csa2
