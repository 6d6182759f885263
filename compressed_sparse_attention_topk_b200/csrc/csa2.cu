// C ABI of the CSA2 hot path (see include/csa2.h for the contract of every
// entry point).  One translation unit: every kernel of the library is
// included here so that they share the device status word.
#include "csa2.h"

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "attn_cluster.cuh"
#include "attn_handoff.cuh"
#include "attn_rows.cuh"
#include "common.cuh"
#include "stage.cuh"
#include "decode_fused.cuh"
#include "index_scan.cuh"
#include "pack.cuh"
#include "pool.cuh"
#include "prefill_gemm.cuh"
#include "row_cluster.cuh"

using namespace csa2;

namespace {

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static std::atomic<int> cache[256];  // per device: 0 unknown
  if (dev >= 0 && dev < 256) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c) return c;
  }
  int v = 148;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) v = 148;
  if (dev >= 0 && dev < 256) cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

csa2_status after_launch() { return cudaGetLastError() == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA; }

// ---------------------------------------------------------------------------
// Kernel timing trace: event pairs around launches while enabled.
// ---------------------------------------------------------------------------
struct TraceRecord {
  const char *name;
  cudaEvent_t start, stop;
};
constexpr size_t kTraceMax = size_t(1) << 16;
bool g_trace_on = false;
TraceRecord *g_trace = nullptr;
size_t g_trace_n = 0;

void trace_clear() {
  for (size_t i = 0; i < g_trace_n; ++i) {
    cudaEventDestroy(g_trace[i].start);
    cudaEventDestroy(g_trace[i].stop);
  }
  g_trace_n = 0;
}

// Records an event on `st`; while `st` is being captured into a CUDA graph
// the record becomes an event-record node of the graph (timed on every
// replay) instead of a capture-internal dependency.
inline void trace_record(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, st);
}

// Brackets one launch: records `start` on construction and `stop` on
// destruction when the trace is on and has room.
struct TraceScope {
  TraceRecord *rec = nullptr;
  cudaStream_t st;
  TraceScope(const char *name, cudaStream_t s) : st(s) {
    if (!g_trace_on || g_trace_n >= kTraceMax) return;
    if (!g_trace) g_trace = new TraceRecord[kTraceMax];
    TraceRecord &r = g_trace[g_trace_n];
    if (cudaEventCreate(&r.start) != cudaSuccess) return;
    if (cudaEventCreate(&r.stop) != cudaSuccess) {
      cudaEventDestroy(r.start);
      return;
    }
    r.name = name;
    rec = &r;
    ++g_trace_n;
    trace_record(r.start, st);
  }
  ~TraceScope() {
    if (rec) trace_record(rec->stop, st);
  }
};

// ---------------------------------------------------------------------------
// Index + top-k: shapes, workspace, launches.
// ---------------------------------------------------------------------------
constexpr int64_t kTopkWsRowBudget = int64_t(1) << 30;  // bytes of per-row scratch per pass
constexpr int64_t kMaxRowsPerPass = 32768;

bool scan_shape_supported(int32_t H_I, int32_t d_I) {
  const bool hi_ok = H_I == 1 || H_I == 2 || H_I == 4 || H_I == 8;
  const bool di_ok = d_I == 16 || d_I == 32 || d_I == 64 || d_I == 128;
  return hi_ok && di_ok && H_I * (d_I / 16) <= 32;
}

int64_t topk_rows_per_pass(int64_t rows, int64_t N) {
  const int64_t per_row = 12 * std::max<int64_t>(N, 1);
  int64_t R = std::max<int64_t>(1, kTopkWsRowBudget / per_row);
  R = std::min<int64_t>(R, kMaxRowsPerPass);
  return std::min<int64_t>(R, std::max<int64_t>(rows, 1));
}

// Row stride of the workspace score rows: a multiple of 4 floats, so every
// row starts 16-byte aligned for bulk copies.
inline int64_t score_stride(int64_t N) { return (N + 3) & ~int64_t(3); }

struct TopkWs {
  float *scores;
  uint2 *cand;
  uint32_t *hist1;
  size_t bytes;
};

TopkWs topk_ws_layout(void *base, int64_t R, int64_t N) {
  TopkWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  const size_t o_scores = take(size_t(R) * score_stride(N) * 4);
  const size_t o_cand = take(size_t(R) * N * 8);
  const size_t o_hist = take(size_t(R) * kHistStride * 4);
  char *p = static_cast<char *>(base);
  w.scores = reinterpret_cast<float *>(p + o_scores);
  w.cand = reinterpret_cast<uint2 *>(p + o_cand);
  w.hist1 = reinterpret_cast<uint32_t *>(p + o_hist);
  w.bytes = off;
  return w;
}

// A decode layer's selection handed to the attention kernel (after the
// top-k workspace): each selecting CTA's list [R][16][topk] and each
// attention CTA's partial per head [R][16][H][D + 4].
struct HandoffWs {
  int32_t *lists;
  float *part;
  size_t bytes;
};

HandoffWs handoff_layout(void *base, int64_t R, int32_t topk, int32_t H, int32_t D) {
  HandoffWs w{};
  const size_t o_lists = 0;
  const size_t o_part = align_up(size_t(R) * ah::kMaxG * topk * 4, 256);
  w.bytes = o_part + align_up(size_t(R) * ah::kMaxG * H * (D + 4) * 4, 256);
  char *p = static_cast<char *>(base);
  w.lists = reinterpret_cast<int32_t *>(p + o_lists);
  w.part = reinterpret_cast<float *>(p + o_part);
  return w;
}

// Per-device one-time kernel attribute setup (dynamic shared memory above
// 48 KiB, non-portable cluster size).  Must run before any stream capture;
// the entry points call it on their first use on a device.
template <typename K>
csa2_status set_smem_attr(K kernel, size_t bytes, bool big_cluster) {
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess)
    return CSA2_ERR_CUDA;
  if (big_cluster &&
      cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
          cudaSuccess)
    return CSA2_ERR_CUDA;
  return CSA2_OK;
}

// Index-key format of a scan: int8 keys, or FP4 keys (k_exps != nullptr).
template <int DI, int HI, int KF>
void launch_scan_kf(dim3 grid, cudaStream_t st, const int8_t *q_idx, const float *w,
                    const int8_t *k_idx, const uint8_t *k_exps, int32_t T, int64_t N,
                    int64_t n_prior, int32_t ratio, int64_t row0, float *scores, int64_t stride,
                    uint32_t *hist1, int write_masked) {
  using S = ScanShape<DI, HI, KF>;
  static std::atomic<bool> done[256];  // per device: attributes set
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 256 || !done[dev].load(std::memory_order_acquire)) {
    set_smem_attr(index_scan_kernel<DI, HI, KF>, S::SMEM, false);
    if (dev >= 0 && dev < 256) done[dev].store(true, std::memory_order_release);
  }
  index_scan_kernel<DI, HI, KF><<<grid, kScanThreads, S::SMEM, st>>>(
      q_idx, w, k_idx, k_exps, T, N, n_prior, ratio, row0, scores, stride, hist1, write_masked,
      ScanBlockMax{});
}

// The int8-key scan that also takes a Full row's block maxima (ScanBlockMax).
template <int DI, int HI>
void launch_scan_bm(dim3 grid, cudaStream_t st, const int8_t *q_idx, const float *w,
                    const int8_t *k_idx, int64_t N, int64_t row0, float *scores, int64_t stride,
                    uint32_t *hist1, const ScanBlockMax &bm) {
  using S = ScanShape<DI, HI, kScanKeysInt8>;
  static std::atomic<bool> done[256];  // per device: attributes set
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 256 || !done[dev].load(std::memory_order_acquire)) {
    set_smem_attr(index_scan_kernel<DI, HI, kScanKeysInt8, true>, S::SMEM, false);
    if (dev >= 0 && dev < 256) done[dev].store(true, std::memory_order_release);
  }
  index_scan_kernel<DI, HI, kScanKeysInt8, true><<<grid, kScanThreads, S::SMEM, st>>>(
      q_idx, w, k_idx, nullptr, 1, N, -1, 1, row0, scores, stride, hist1, 0, bm);
}

template <int DI, int HI>
void launch_scan(dim3 grid, cudaStream_t st, const int8_t *q_idx, const float *w,
                 const int8_t *k_idx, int32_t T, int64_t N, int64_t n_prior, int32_t ratio,
                 int64_t row0, float *scores, int64_t stride, uint32_t *hist1,
                 int write_masked) {
  launch_scan_kf<DI, HI, kScanKeysInt8>(grid, st, q_idx, w, k_idx, nullptr, T, N, n_prior, ratio,
                                        row0, scores, stride, hist1, write_masked);
}

using ScanLaunch = void (*)(dim3, cudaStream_t, const int8_t *, const float *, const int8_t *,
                            int32_t, int64_t, int64_t, int32_t, int64_t, float *, int64_t,
                            uint32_t *, int);
using ScanLaunchFp4 = void (*)(dim3, cudaStream_t, const int8_t *, const float *, const int8_t *,
                               const uint8_t *, int32_t, int64_t, int64_t, int32_t, int64_t,
                               float *, int64_t, uint32_t *, int);

using ScanLaunchBM = void (*)(dim3, cudaStream_t, const int8_t *, const float *, const int8_t *,
                              int64_t, int64_t, float *, int64_t, uint32_t *,
                              const ScanBlockMax &);

// Decode shapes whose scan also takes the block maxima of a Full layer's pool.
ScanLaunchBM pick_scan_bm(int32_t d_I, int32_t H_I) {
  if (d_I == 32 && H_I == 4) return &launch_scan_bm<32, 4>;
  if (d_I == 64 && H_I == 4) return &launch_scan_bm<64, 4>;
  return nullptr;
}

ScanLaunchFp4 pick_scan_fp4(int32_t d_I, int32_t H_I) {
  if (d_I == 32 && H_I == 4) return &launch_scan_kf<32, 4, kScanKeysFp4>;
  if (d_I == 64 && H_I == 4) return &launch_scan_kf<64, 4, kScanKeysFp4>;
  return nullptr;
}

ScanLaunch pick_scan(int32_t d_I, int32_t H_I) {
#define CSA2_SCAN_CASE(DI, HI) \
  if (d_I == DI && H_I == HI) return &launch_scan<DI, HI>;
  CSA2_SCAN_CASE(16, 1) CSA2_SCAN_CASE(16, 2) CSA2_SCAN_CASE(16, 4) CSA2_SCAN_CASE(16, 8)
  CSA2_SCAN_CASE(32, 1) CSA2_SCAN_CASE(32, 2) CSA2_SCAN_CASE(32, 4) CSA2_SCAN_CASE(32, 8)
  CSA2_SCAN_CASE(64, 1) CSA2_SCAN_CASE(64, 2) CSA2_SCAN_CASE(64, 4) CSA2_SCAN_CASE(64, 8)
  CSA2_SCAN_CASE(128, 1) CSA2_SCAN_CASE(128, 2) CSA2_SCAN_CASE(128, 4)
#undef CSA2_SCAN_CASE
  return nullptr;
}

template <int DI, int HI, int TQ>
void launch_scan_group(dim3 grid, cudaStream_t st, const int8_t *q_idx, const float *w,
                       const int8_t *k_idx, int32_t T, int64_t N, int64_t n_prior, int32_t ratio,
                       int64_t row0, float *scores, int64_t stride, uint32_t *hist1,
                       int write_masked) {
  using S = ScanGroupShape<DI, HI, TQ>;
  static std::atomic<bool> done[256];  // per device: attributes set
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 256 || !done[dev].load(std::memory_order_acquire)) {
    set_smem_attr(index_scan_group_kernel<DI, HI, TQ>, S::SMEM, false);
    if (dev >= 0 && dev < 256) done[dev].store(true, std::memory_order_release);
  }
  index_scan_group_kernel<DI, HI, TQ><<<grid, S::THREADS, S::SMEM, st>>>(
      q_idx, w, k_idx, T, N, n_prior, ratio, row0, scores, stride, hist1, write_masked);
}

template <int DI, int TQ>
void launch_scan_mma(dim3 grid, cudaStream_t st, const int8_t *q_idx, const float *w,
                     const int8_t *k_idx, int32_t T, int64_t N, int64_t n_prior, int32_t ratio,
                     int64_t row0, float *scores, int64_t stride, uint32_t *hist1,
                     int write_masked) {
  using S = ScanMmaShape<DI, TQ>;
  static std::atomic<bool> done[256];  // per device: attributes set
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 256 || !done[dev].load(std::memory_order_acquire)) {
    set_smem_attr(index_scan_mma_kernel<DI, TQ>, S::smem(TQ), false);
    if (dev >= 0 && dev < 256) done[dev].store(true, std::memory_order_release);
  }
  index_scan_mma_kernel<DI, TQ><<<grid, S::THREADS, S::smem(T), st>>>(
      q_idx, w, k_idx, T, N, n_prior, ratio, row0, scores, stride, hist1, write_masked);
}

// Several query rows per sequence (2 <= T <= 8, d_I <= 64): one scan of the
// keys serves all of them; with 4 index heads and d_I in {32, 64} the dots
// run on the tensor cores (index_scan_mma_kernel).
ScanLaunch pick_scan_group(int32_t d_I, int32_t H_I, int32_t T) {
  if (T < 2 || T > 8 || d_I > 64) return nullptr;
  if (H_I == 4 && (d_I == 32 || d_I == 64)) {
    if (d_I == 32) return T <= 2 ? &launch_scan_mma<32, 2> : T <= 4 ? &launch_scan_mma<32, 4>
                                                                    : &launch_scan_mma<32, 8>;
    return T <= 2 ? &launch_scan_mma<64, 2> : T <= 4 ? &launch_scan_mma<64, 4>
                                                     : &launch_scan_mma<64, 8>;
  }
#define CSA2_SG_CASE(DI, HI)                                                    \
  if (d_I == DI && H_I == HI) {                                                 \
    if (T <= 2) return &launch_scan_group<DI, HI, 2>;                           \
    if (T <= 4) return &launch_scan_group<DI, HI, 4>;                           \
    return &launch_scan_group<DI, HI, 8>;                                       \
  }
  CSA2_SG_CASE(16, 1) CSA2_SG_CASE(16, 2) CSA2_SG_CASE(16, 4) CSA2_SG_CASE(16, 8)
  CSA2_SG_CASE(32, 1) CSA2_SG_CASE(32, 2) CSA2_SG_CASE(32, 4) CSA2_SG_CASE(32, 8)
  CSA2_SG_CASE(64, 1) CSA2_SG_CASE(64, 2) CSA2_SG_CASE(64, 4) CSA2_SG_CASE(64, 8)
#undef CSA2_SG_CASE
  return nullptr;
}

// ---- the per-row cluster kernel -------------------------------------------
template <int D, int CL, bool HO = false>
csa2_status launch_row_cl(const RowParams &p, int64_t nr, cudaStream_t st) {
  const size_t smem = sizeof(RowSmem<D>);
  static std::atomic<bool> done[256];  // per device: attributes set
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 256 || !done[dev].load(std::memory_order_acquire)) {
    if (set_smem_attr(row_cluster_kernel<D, CL, HO>, smem, CL > 8) != CSA2_OK)
      return CSA2_ERR_CUDA;
    if (dev >= 0 && dev < 256) done[dev].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nr * CL), 1, 1);
  cfg.blockDim = dim3(kRowThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // After a scan, start early: the kernel waits for the scan's results itself.
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.do_topk ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, row_cluster_kernel<D, CL, HO>, p) == cudaSuccess
             ? CSA2_OK
             : CSA2_ERR_CUDA;
}

// Clusters of cl CTAs of `kernel` (threads per CTA, dynamic shared memory
// smem) that this device can hold at once; 0 when none can be launched.
template <class K>
int max_active_clusters(K kernel, int cl, int threads, size_t smem) {
  if (set_smem_attr(kernel, smem, cl > 8) != CSA2_OK) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)cl, 1, 1);
  cfg.blockDim = dim3((unsigned)threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// The row kernel's resident clusters of CL CTAs (cached per device).
template <int D, int CL>
int row_clusters_resident() {
  static std::atomic<int> cache[256];  // per device: 0 unknown, else count + 1
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 256) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c) return c - 1;
  }
  const int n = max_active_clusters(row_cluster_kernel<D, CL, false>, CL, kRowThreads,
                                    sizeof(RowSmem<D>));
  if (dev >= 0 && dev < 256) cache[dev].store(n + 1, std::memory_order_relaxed);
  return n;
}

// Rows of one launch -> CTAs per row: the largest cluster (16, 8 or 4 CTAs)
// whose clusters for all nr rows the device holds at once, so that no row's
// cluster waits for another's to finish (4 when neither fits).  A second
// wave costs a whole selection: 32 decode rows take 80 us per step in
// clusters of 8 (256 CTAs for 148 SMs) and 68 us in clusters of 4.
int row_cluster_size(int64_t nr, int D) {
  if (nr <= (D == 128 ? row_clusters_resident<128, 16>() : row_clusters_resident<64, 16>()))
    return 16;
  if (nr <= (D == 128 ? row_clusters_resident<128, 8>() : row_clusters_resident<64, 8>()))
    return 8;
  return 4;
}

csa2_status launch_row(const RowParams &p, int D, int64_t nr, cudaStream_t st) {
  TraceScope ts(p.do_topk ? (p.do_attn ? "topk_attend" : "topk_select") : "attend", st);
  const int cl = row_cluster_size(nr, D);
  if (p.lists) {  // hand-off instances: 8 or fewer CTAs per row
    if (p.do_attn || !p.do_topk || cl > 8) return CSA2_ERR_UNSUPPORTED;
    if (D == 128)
      return cl == 8 ? launch_row_cl<128, 8, true>(p, nr, st) : launch_row_cl<128, 4, true>(p, nr, st);
    return cl == 8 ? launch_row_cl<64, 8, true>(p, nr, st) : launch_row_cl<64, 4, true>(p, nr, st);
  }
  if (D == 128) {
    if (cl == 16) return launch_row_cl<128, 16>(p, nr, st);
    if (cl == 8) return launch_row_cl<128, 8>(p, nr, st);
    return launch_row_cl<128, 4>(p, nr, st);
  }
  if (cl == 16) return launch_row_cl<64, 16>(p, nr, st);
  if (cl == 8) return launch_row_cl<64, 8>(p, nr, st);
  return launch_row_cl<64, 4>(p, nr, st);
}

// ---- the per-row attention cluster kernel (attn_cluster.cuh) --------------
template <int D, int CL>
csa2_status launch_attn_cl(const ar::Params &a, int64_t nr, bool after_topk, cudaStream_t st) {
  const size_t smem = sizeof(ac::Smem<D, CL>);
  static std::atomic<bool> done[256];  // per device: attributes set
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 256 || !done[dev].load(std::memory_order_acquire)) {
    if (set_smem_attr(ac::attn_cluster_kernel<D, CL>, smem, CL > 8) != CSA2_OK)
      return CSA2_ERR_CUDA;
    if (dev >= 0 && dev < 256) done[dev].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nr * CL), 1, 1);
  cfg.blockDim = dim3(ac::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // After the selection, start early: the kernel loads the query and
  // attends over the window, then waits for the selection's results itself.
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_topk ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, ac::attn_cluster_kernel<D, CL>, a, after_topk ? 1 : 0) ==
                 cudaSuccess
             ? CSA2_OK
             : CSA2_ERR_CUDA;
}

// The attention cluster kernel's resident clusters of CL CTAs (cached per
// device).
template <int D, int CL>
int attn_clusters_resident() {
  static std::atomic<int> cache[256];  // per device: 0 unknown, else count + 1
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 256) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c) return c - 1;
  }
  const int n = max_active_clusters(ac::attn_cluster_kernel<D, CL>, CL, ac::kThreads,
                                    sizeof(ac::Smem<D, CL>));
  if (dev >= 0 && dev < 256) cache[dev].store(n + 1, std::memory_order_relaxed);
  return n;
}

// Attention of nr decode rows (a.row0 ...): CTAs per row as for the
// selection; after_topk: launched right
// after the selection of the same rows, with programmatic dependent launch.
csa2_status launch_attn_cluster(const ar::Params &a, int D, int64_t nr, bool after_topk,
                                cudaStream_t st) {
  TraceScope ts("attend", st);
  // the largest cluster whose clusters for all the rows are resident at once
  int cl = 4;
  if (nr <= (D == 128 ? attn_clusters_resident<128, 16>() : attn_clusters_resident<64, 16>()))
    cl = 16;
  else if (nr <= (D == 128 ? attn_clusters_resident<128, 8>() : attn_clusters_resident<64, 8>()))
    cl = 8;
  if (D == 128) {
    if (cl == 16) return launch_attn_cl<128, 16>(a, nr, after_topk, st);
    if (cl == 8) return launch_attn_cl<128, 8>(a, nr, after_topk, st);
    return launch_attn_cl<128, 4>(a, nr, after_topk, st);
  }
  if (cl == 16) return launch_attn_cl<64, 16>(a, nr, after_topk, st);
  if (cl == 8) return launch_attn_cl<64, 8>(a, nr, after_topk, st);
  return launch_attn_cl<64, 4>(a, nr, after_topk, st);
}

// ---- the attention kernel fed by the selection (attn_handoff.cuh) ---------
template <int D>
csa2_status launch_attn_handoff_d(const ah::Params &hp, int64_t nr, cudaStream_t st) {
  const size_t smem = sizeof(ah::Smem<D>);
  static std::atomic<bool> done[256];  // per device: attributes set
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 256 || !done[dev].load(std::memory_order_acquire)) {
    if (set_smem_attr(ah::attn_handoff_kernel<D>, smem, false) != CSA2_OK) return CSA2_ERR_CUDA;
    if (dev >= 0 && dev < 256) done[dev].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nr * hp.G), 1, 1);
  cfg.blockDim = dim3(ah::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  // Start early (programmatic dependent launch): the kernel loads the query
  // and attends over the window, then waits for each list's ready flag.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, ah::attn_handoff_kernel<D>, hp) == cudaSuccess ? CSA2_OK
                                                                                  : CSA2_ERR_CUDA;
}

csa2_status launch_attn_handoff(const ah::Params &hp, int D, int64_t nr, cudaStream_t st) {
  TraceScope ts("attend_handoff", st);
  if (hp.G < 1 || hp.G > ah::kMaxG || hp.G > kHandoffFlags) return CSA2_ERR_UNSUPPORTED;
  return D == 128 ? launch_attn_handoff_d<128>(hp, nr, st) : launch_attn_handoff_d<64>(hp, nr, st);
}

csa2_status check_topk_args(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B,
                            int32_t T, int32_t H_I, int32_t d_I, int64_t N, int64_t n_prior,
                            int32_t ratio, int32_t topk, const int32_t *idx_out,
                            const float *score_out) {
  if (B < 0 || T < 0 || N < 0 || topk < 1 || H_I < 1 || d_I < 1) return CSA2_ERR_INVALID_ARG;
  if (n_prior >= 0 && ratio < 1) return CSA2_ERR_INVALID_ARG;
  if (d_I % 16 != 0) return CSA2_ERR_INVALID_ARG;
  if (!scan_shape_supported(H_I, d_I) || topk > 65536 || N >= (int64_t(1) << 31) - 1)
    return CSA2_ERR_UNSUPPORTED;
  if (int64_t(B) * T == 0) return CSA2_OK;
  if (!q_idx || !w || !idx_out || (N > 0 && !k_idx)) return CSA2_ERR_INVALID_ARG;
  if (!aligned(q_idx, 16) || (k_idx && !aligned(k_idx, 16)) || !aligned(w, 4) ||
      !aligned(idx_out, 4) || (score_out && !aligned(score_out, 4)))
    return CSA2_ERR_INVALID_ARG;
  return CSA2_OK;
}

size_t topk_ws_bytes(int32_t B, int32_t T, int64_t N) {
  const int64_t rows = int64_t(B) * T;
  const int64_t R = topk_rows_per_pass(rows, N);
  return topk_ws_layout(nullptr, R, N).bytes;
}

// ---------------------------------------------------------------------------
// Chunked prefill on the tensor cores (see prefill_gemm.cuh): shapes,
// workspace, tensor maps and the per-pass launch sequence.
// ---------------------------------------------------------------------------
constexpr int64_t kPfMinT = 64;  // below this many queries per sequence the per-row scan is used

int pf_cap(int32_t topk) { return std::max(8192, 4 * topk); }

bool pf_eligible(int32_t T, int32_t H_I, int32_t d_I, int64_t N, int32_t topk,
                 const float *score_out);

struct PfWs {
  int8_t *qa;
  double *sigma, *err;
  int32_t *tau, *fail_rows, *fail_count;
  int32_t *smp;
  uint32_t *bits;
  int64_t smp_pitch, bits_pitch;
  size_t bytes;
};

PfWs pf_ws_layout(void *base, int64_t R, int64_t N, int32_t d_I) {
  PfWs w{};
  w.smp_pitch = pf::kSampleMax;
  w.bits_pitch = align_up(size_t(ceil_div(N, 32)), 32);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  const size_t o_qa = take(size_t(R) * 2 * d_I);
  const size_t o_sigma = take(size_t(R) * 8);
  const size_t o_err = take(size_t(R) * 8);
  const size_t o_tau = take(size_t(R) * 4);
  const size_t o_fail = take(size_t(R) * 4);
  const size_t o_failn = take(4);
  const size_t o_smp = take(size_t(R) * w.smp_pitch * 4);
  const size_t o_bits = take(size_t(R) * w.bits_pitch * 4);
  char *p = static_cast<char *>(base);
  w.qa = reinterpret_cast<int8_t *>(p + o_qa);
  w.sigma = reinterpret_cast<double *>(p + o_sigma);
  w.err = reinterpret_cast<double *>(p + o_err);
  w.tau = reinterpret_cast<int32_t *>(p + o_tau);
  w.fail_rows = reinterpret_cast<int32_t *>(p + o_fail);
  w.fail_count = reinterpret_cast<int32_t *>(p + o_failn);
  w.smp = reinterpret_cast<int32_t *>(p + o_smp);
  w.bits = reinterpret_cast<uint32_t *>(p + o_bits);
  w.bytes = off;
  return w;
}

// Query rows per pass: a multiple of 128 within the per-pass budget.
int64_t pf_rows_per_pass(int32_t T, int64_t N, int32_t d_I) {
  const int64_t per_row =
      2 * d_I + 32 + int64_t(pf::kSampleMax) * 4 + int64_t(align_up(size_t(ceil_div(N, 32)), 32)) * 4;
  int64_t R = std::max<int64_t>(pf::kQ, kTopkWsRowBudget / per_row / pf::kQ * pf::kQ);
  return std::min<int64_t>(R, ceil_div(T, pf::kQ) * pf::kQ);
}

size_t pf_ws_bytes(int32_t T, int64_t N, int32_t d_I) {
  return pf_ws_layout(nullptr, pf_rows_per_pass(T, N, d_I), N, d_I).bytes;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on the driver library).
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = [] {  // looked up once (thread-safe initialisation)
    EncodeTiledFn f = nullptr;
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f = reinterpret_cast<EncodeTiledFn>(ptr);
    cudaGetLastError();
    return f;
  }();
  return fn;
}

// 3-D byte tensor map: dims {d0, d1, d2}, byte strides of dims 1 and 2, box
// {d0, b1, b2}, swizzled over d0 bytes (d0 in {32, 64, 128}).
bool make_map_u8(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint64_t s1, uint64_t s2, uint32_t b1, uint32_t b2) {
  EncodeTiledFn f = encode_tiled();
  if (!f || d1 == 0 || d2 == 0) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1, s2};
  const cuuint32_t box[3] = {(cuuint32_t)d0, b1, b2};
  const cuuint32_t es[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = d0 == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : d0 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                           : CU_TENSOR_MAP_SWIZZLE_32B;
  return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shapes the tensor-core prefill path serves (host arithmetic only: the
// workspace query answers the same with or without a GPU driver).
bool pf_shape_ok(int32_t T, int32_t H_I, int32_t d_I, int64_t N, int32_t topk) {
  return T >= kPfMinT && (d_I == 32 || d_I == 64 || d_I == 128) &&
         scan_shape_supported(H_I, d_I) && N >= 1 && N < (int64_t(1) << 31) - 1 &&
         4 * int64_t(topk) <= 16384;
}

bool pf_eligible(int32_t T, int32_t H_I, int32_t d_I, int64_t N, int32_t topk,
                 const float *score_out) {
  return pf_shape_ok(T, H_I, d_I, N, topk) && score_out == nullptr && encode_tiled() != nullptr;
}

// Key-axis positions per CTA: minimises (waves of CTAs) x (tiles per CTA +
// a fixed per-CTA cost), over multiples of the staging unit.
int64_t pf_split_len(int64_t axis, int64_t nblk, int sms) {
  const int64_t units = std::max<int64_t>(1, ceil_div(axis, pf::kAxisUnit));
  int64_t best_len = units * pf::kAxisUnit, best_cost = INT64_MAX;
  for (int64_t ns = 1; ns <= units; ++ns) {
    const int64_t len = ceil_div(units, ns) * pf::kAxisUnit;
    const int64_t nsplit = ceil_div(axis, len);
    const int64_t waves = ceil_div(nblk * nsplit, sms);
    const int64_t cost = waves * (len / pf::kN + 6);
    if (cost < best_cost) {
      best_cost = cost;
      best_len = len;
    }
  }
  return best_len;
}

template <int DI, bool SAMPLE>
csa2_status launch_pf_gemm(const CUtensorMap &amap, const CUtensorMap &bmap,
                           const pf::GemmParams &p, int64_t nsplit, int64_t nblk,
                           cudaStream_t st) {
  const size_t smem = pf::gemm_smem_bytes<DI>();
  static std::atomic<bool> done[256];  // per device: attributes set
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 256 || !done[dev].load(std::memory_order_acquire)) {
    if (set_smem_attr(pf::pf_gemm_kernel<DI, SAMPLE>, smem, false) != CSA2_OK)
      return CSA2_ERR_CUDA;
    if (dev >= 0 && dev < 256) done[dev].store(true, std::memory_order_release);
  }
  TraceScope ts(SAMPLE ? "pf_sample_mma" : "pf_filter_mma", st);
  pf::pf_gemm_kernel<DI, SAMPLE>
      <<<dim3((unsigned)nsplit, (unsigned)nblk), pf::kGemmThreads, smem, st>>>(amap, bmap, p);
  return after_launch();
}

template <int DI, int HI>
csa2_status pf_run_rows(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B,
                        int32_t T, int64_t N, int64_t n_prior, int32_t ratio, int32_t topk,
                        int32_t *idx_out, const PfWs &L, int64_t R, cudaStream_t st) {
  const int sms = device_sms();
  const int cap = pf_cap(topk);
  const size_t sel_smem = pf::sel_head_bytes<DI, HI>() + size_t(cap) * 8;
  {
    static std::atomic<bool> done[256];  // per device: attributes set
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 256 || !done[dev].load(std::memory_order_acquire)) {
      if (set_smem_attr(pf::pf_select_kernel<DI, HI>, pf::sel_head_bytes<DI, HI>() + 16384 * 8,
                        false) != CSA2_OK)
        return CSA2_ERR_CUDA;
      if (dev >= 0 && dev < 256) done[dev].store(true, std::memory_order_release);
    }
  }
  CUtensorMap kmap;
  if (!make_map_u8(&kmap, k_idx, DI, uint64_t(N), uint64_t(B), DI, uint64_t(N) * DI, pf::kN, 1))
    return CSA2_ERR_CUDA;
  for (int32_t b = 0; b < B; ++b) {
    for (int32_t t0 = 0; t0 < T; t0 += (int32_t)R) {
      const int32_t tc = (int32_t)std::min<int64_t>(R, T - t0);
      const int64_t nblk = ceil_div(tc, pf::kQ);
      const int64_t vmax = pf::visible_count(N, n_prior, ratio, (int64_t)t0 + tc - 1);
      if (cudaMemsetAsync(L.fail_count, 0, 4, st) != cudaSuccess) return CSA2_ERR_CUDA;
      {
        TraceScope ts("pf_prep", st);
        pf::pf_prep_kernel<DI, HI><<<(unsigned)ceil_div(tc, 8), 256, 0, st>>>(
            q_idx, w, T, b, t0, tc, L.qa, L.sigma, L.err);
        if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
      }
      CUtensorMap amap;
      if (!make_map_u8(&amap, L.qa, DI, 2, uint64_t(tc), DI, 2 * DI, 1, pf::kQ))
        return CSA2_ERR_CUDA;
      pf::GemmParams gp{};
      gp.N = N;
      gp.T = T;
      gp.n_prior = n_prior;
      gp.ratio = ratio;
      gp.b = b;
      gp.t_begin = t0;
      gp.t_count = tc;
      gp.level_scale = 256;
      // sample pass (only needed when some row has more visible entries
      // than the selection capacity)
      const int32_t sstride =
          (int32_t)std::max<int64_t>(1, ceil_div(std::max<int64_t>(vmax, 1), pf::kSampleMax));
      const int64_t nsamp = ceil_div(std::max<int64_t>(vmax, 1), sstride);
      if (vmax > cap) {
        CUtensorMap smap;
        const uint64_t seq_samples = uint64_t(ceil_div(N, sstride));
        if (!make_map_u8(&smap, k_idx, DI, seq_samples, uint64_t(B), uint64_t(sstride) * DI,
                         uint64_t(N) * DI, pf::kN, 1))
          return CSA2_ERR_CUDA;
        gp.sstride = sstride;
        gp.smp = L.smp;
        gp.smp_pitch = L.smp_pitch;
        gp.axis_len = nsamp;
        gp.split_len = pf_split_len(nsamp, nblk, sms);
        const int64_t nsplit = ceil_div(nsamp, gp.split_len);
        if (launch_pf_gemm<DI, true>(amap, smap, gp, nsplit, nblk, st) != CSA2_OK)
          return CSA2_ERR_CUDA;
      }
      {
        pf::ThetaParams tp{};
        tp.N = N;
        tp.n_prior = n_prior;
        tp.ratio = ratio;
        tp.t_begin = t0;
        tp.t_count = tc;
        tp.sstride = sstride;
        tp.nsamp = nsamp;
        tp.smp = L.smp;
        tp.smp_pitch = L.smp_pitch;
        tp.target = 2 * topk;
        tp.cap = cap;
        tp.sigma = L.sigma;
        tp.err = L.err;
        tp.tau = L.tau;
        TraceScope ts("pf_theta", st);
        pf::pf_theta_kernel<<<(unsigned)tc, pf::kThetaThreads, 0, st>>>(tp);
        if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
      }
      gp.axis_len = vmax;
      gp.split_len = pf_split_len(vmax, nblk, sms);
      gp.tau = L.tau;
      gp.bits = L.bits;
      gp.bits_pitch = L.bits_pitch;
      gp.sstride = 1;
      gp.smp = nullptr;
      {
        const int64_t nsplit = ceil_div(std::max<int64_t>(vmax, 1), gp.split_len);
        if (launch_pf_gemm<DI, false>(amap, kmap, gp, nsplit, nblk, st) != CSA2_OK)
          return CSA2_ERR_CUDA;
      }
      pf::SelParams sp{};
      sp.q_idx = q_idx;
      sp.w = w;
      sp.k_idx = k_idx;
      sp.N = N;
      sp.T = T;
      sp.n_prior = n_prior;
      sp.ratio = ratio;
      sp.b = b;
      sp.t_begin = t0;
      sp.t_count = tc;
      sp.topk = topk;
      sp.cap = cap;
      sp.bits = L.bits;
      sp.bits_pitch = L.bits_pitch;
      sp.tau = L.tau;
      sp.sigma = L.sigma;
      sp.err = L.err;
      sp.idx = idx_out;
      sp.fail_rows = L.fail_rows;
      sp.fail_count = L.fail_count;
      {
        TraceScope ts("pf_select", st);
        pf::pf_select_kernel<DI, HI><<<(unsigned)tc, pf::kSelThreads, sel_smem, st>>>(sp);
        if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
      }
      {
        TraceScope ts("pf_fallback", st);
        pf::pf_fallback_kernel<DI, HI>
            <<<(unsigned)std::min<int64_t>(tc, sms), pf::kSelThreads, 0, st>>>(sp);
        if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
      }
    }
  }
  return CSA2_OK;
}

using PfRun = csa2_status (*)(const int8_t *, const float *, const int8_t *, int32_t, int32_t,
                              int64_t, int64_t, int32_t, int32_t, int32_t *, const PfWs &,
                              int64_t, cudaStream_t);

PfRun pick_pf(int32_t d_I, int32_t H_I) {
#define CSA2_PF_CASE(DI, HI) \
  if (d_I == DI && H_I == HI) return &pf_run_rows<DI, HI>;
  CSA2_PF_CASE(32, 1) CSA2_PF_CASE(32, 2) CSA2_PF_CASE(32, 4) CSA2_PF_CASE(32, 8)
  CSA2_PF_CASE(64, 1) CSA2_PF_CASE(64, 2) CSA2_PF_CASE(64, 4) CSA2_PF_CASE(64, 8)
  CSA2_PF_CASE(128, 1) CSA2_PF_CASE(128, 2) CSA2_PF_CASE(128, 4)
#undef CSA2_PF_CASE
  return nullptr;
}

struct AttnArgs {  // attention inputs of one layer (all device pointers)
  const uint16_t *q;
  const uint8_t *codes;
  const float *scales;
  const uint16_t *win_k, *win_v;
  int32_t H, D, W;
  float sm_scale;
  float *out, *lse;
};

csa2_status run_attn(const uint16_t *q, const uint8_t *codes, const float *scales,
                     const int32_t *idx, const uint16_t *win_k, const uint16_t *win_v, int32_t B,
                     int32_t T, int32_t H, int32_t D, int64_t N, int32_t topk, int32_t W,
                     float sm_scale, float *out, float *lse, cudaStream_t st);

// ---------------------------------------------------------------------------
// The fused decode layer kernel (decode_fused.cuh): decode rows (one query
// per sequence, every entry visible), no score output.
// ---------------------------------------------------------------------------
constexpr int kFusedMaxP = fd::kMaxP;                 // attention CTAs per row
constexpr int64_t kFusedMaxRows = fd::kMaxG / 4;      // rows per launch (at least 4 CTAs each)
constexpr int kFusedMaxPartD = 128;

// Which kernels serve decode rows (csa2_set_decode_kernel): the index scan
// + per-row cluster kernel (default), or the fused single-launch kernel.
// The environment variable CSA2_DECODE_KERNEL=fused sets the initial choice.
std::atomic<int> g_decode_kernel{-1};

bool fused_enabled() {
  int v = g_decode_kernel.load(std::memory_order_relaxed);
  if (v < 0) {
    const char *e = std::getenv("CSA2_DECODE_KERNEL");
    v = (e && std::strcmp(e, "fused") == 0) ? CSA2_DECODE_FUSED : CSA2_DECODE_SCAN_CLUSTER;
    g_decode_kernel.store(v, std::memory_order_relaxed);
  }
  return v == CSA2_DECODE_FUSED;
}

struct FusedWs {
  uint32_t *hist1, *arrive, *cnt;
  uint2 *cand;
  float *part;
  size_t sync_bytes, bytes;
};

// Workspace of one launch of R rows: histograms and counters (cleared
// before the launch, contiguous), slice counts, candidate lists, partials.
FusedWs fused_ws_layout(void *base, int64_t R, int64_t N) {
  FusedWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  const size_t o_hist = take(size_t(R) * fd::kHistStride * 4);
  const size_t o_arr = off;  // right after the histograms: one clear covers both
  off = o_arr + align_up(size_t(R) * fd::kArrive * 4, 256);
  w.sync_bytes = off;
  const size_t o_cnt = take(size_t(R) * fd::kMaxG * 4);
  const size_t o_cand = take(size_t(R) * N * 8);
  const size_t o_part = take(size_t(R) * kFusedMaxP * fd::kHeads * (kFusedMaxPartD + 4) * 4);
  char *p = static_cast<char *>(base);
  w.hist1 = reinterpret_cast<uint32_t *>(p + o_hist);
  w.arrive = reinterpret_cast<uint32_t *>(p + o_arr);
  w.cnt = reinterpret_cast<uint32_t *>(p + o_cnt);
  w.cand = reinterpret_cast<uint2 *>(p + o_cand);
  w.part = reinterpret_cast<float *>(p + o_part);
  w.bytes = off;
  return w;
}

size_t fused_ws_bytes(int64_t rows, int64_t N) {
  return fused_ws_layout(nullptr, std::min<int64_t>(rows, kFusedMaxRows), N).bytes;
}

// FP4 index keys: decode rows, d_I in {32, 64}, H_I == 4, N % 16 == 0 (the
// bulk copies of the block exponents start on 16-byte boundaries).
bool fp4_shape_ok(int32_t T, int32_t H_I, int32_t d_I, int64_t N, int64_t n_prior) {
  return T == 1 && n_prior < 0 && (d_I == 32 || d_I == 64) && H_I == 4 && N >= 1 && N % 16 == 0;
}

bool fused_shape_ok(int32_t T, int32_t H_I, int32_t d_I, int64_t N, int64_t n_prior,
                    int32_t topk, bool fp4_keys = false) {
  if (T != 1 || n_prior >= 0 || N < 1 || topk > fd::kSelCap) return false;
  if (fp4_keys)  // bulk copies of the block exponents start on 16-byte boundaries
    return (d_I == 32 || d_I == 64) && H_I == 4 && N % 16 == 0;
  return (d_I == 32 || d_I == 64) && (H_I == 4 || H_I == 8);
}

struct FusedPlan {
  bool ok;
  int G, P, stages, g_row;
  int64_t R, per_cta;
  uint32_t off_sc, off_hist, off_qs, cap;
  size_t dyn;
};

// Launch shape for `rows` rows: rows per launch, CTAs, slice length and the
// shared-memory layout (key ring, the slice's scores, histogram, index
// query; the candidate list and attention buffers reuse the same bytes).
FusedPlan plan_fused(int64_t rows, int64_t N, int32_t d_I, int32_t H_I, int32_t D, int32_t topk,
                     size_t static_smem, int sms, int blocks_per_sm, size_t tile) {
  FusedPlan pl{};
  const size_t maxdyn = size_t(232448) - static_smem - 1024;
  const size_t aw = size_t(fd::kAttnWarps) * (D == 128 ? sizeof(ar::WarpArea<128>)
                                                        : sizeof(ar::WarpArea<64>));
  const int gmax = std::min(sms * std::max(blocks_per_sm, 0), fd::kMaxG);
  for (int64_t R = std::min<int64_t>(rows, std::max(1, gmax / 4)); R >= 1; R = R / 2) {
    // g_row CTAs per row, each scanning one slice of the row (slices never
    // cross rows); at least 16 per row so the attention spreads, at most
    // what fills the SMs
    const int64_t tot = R * N;
    const int64_t G0 = std::min<int64_t>(gmax, std::max<int64_t>(16 * R, ceil_div(tot, 4096)));
    const int g_row = (int)(G0 / R);
    if (g_row < 1) continue;
    const int64_t per = align_up(size_t(ceil_div(N, g_row)), 16);
    const int G = g_row * (int)R;
    const int P = std::min<int>(kFusedMaxP, g_row);
    if (ceil_div(topk, P) > fd::kSelCap) continue;
    const size_t sc = align_up(size_t(per) * 4, 128);
    const size_t fixed = sc + size_t(kBins1) * 4 + align_up(size_t(H_I) * d_I, 128);
    if (fixed + 2 * tile > maxdyn) continue;
    const int stages = (int)std::min<size_t>(4, (maxdyn - fixed) / tile);
    const size_t dyn_a = stages * tile + fixed;
    size_t dyn = std::max(dyn_a, aw);
    dyn = std::max(dyn, size_t(4096) * 8 + size_t(kBins2) * 4);
    if (dyn > maxdyn) continue;
    pl.ok = true;
    pl.G = G;
    pl.g_row = g_row;
    pl.P = P;
    pl.stages = stages;
    pl.R = R;
    pl.per_cta = per;
    pl.off_sc = (uint32_t)(stages * tile);
    pl.off_hist = (uint32_t)(pl.off_sc + sc);
    pl.off_qs = (uint32_t)(pl.off_hist + size_t(kBins1) * 4);
    pl.cap = (uint32_t)((dyn - size_t(kBins2) * 4) / 8);
    pl.dyn = dyn;
    return pl;
  }
  return pl;
}

template <int DI, int HI, int D, int KF>
csa2_status run_fused_t(const fd::Params &base, int64_t rows, cudaStream_t st, void *ws,
                        size_t ws_bytes) {
  auto kern = fd::decode_fused_kernel<DI, HI, D, KF>;
  const size_t tile = fd::Shape<DI, HI, KF>::TILE_BYTES;
  static std::atomic<size_t> static_smem[256];  // per device, set before bps
  static std::atomic<int> bps[256];             // per device: 0 unknown
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 256) return CSA2_ERR_CUDA;
  if (!bps[dev].load(std::memory_order_acquire)) {
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return CSA2_ERR_CUDA;
    const size_t mx = size_t(232448) - fa.sharedSizeBytes - 1024;
    if (set_smem_attr(kern, mx, false) != CSA2_OK) return CSA2_ERR_CUDA;
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, fd::kThreads, mx) !=
        cudaSuccess)
      return CSA2_ERR_CUDA;
    static_smem[dev].store(fa.sharedSizeBytes, std::memory_order_relaxed);
    bps[dev].store(nb > 0 ? nb : -1, std::memory_order_release);
  }
  if (bps[dev] < 1) return CSA2_ERR_UNSUPPORTED;
  const FusedPlan pl = plan_fused(rows, base.N, DI, HI, D, base.topk, static_smem[dev],
                                  device_sms(), bps[dev], tile);
  if (!pl.ok) return CSA2_ERR_UNSUPPORTED;
  const FusedWs L = fused_ws_layout(ws, pl.R, base.N);
  if (!ws || ws_bytes < L.bytes) return CSA2_ERR_WORKSPACE;
  for (int64_t row0 = 0; row0 < rows;) {
    // a launch of q.R rows; the last ones may take fewer rows, with a plan
    // of their own that never holds more rows than the workspace layout
    const int64_t nr = std::min<int64_t>(pl.R, rows - row0);
    const FusedPlan q = nr == pl.R ? pl
                                   : plan_fused(nr, base.N, DI, HI, D, base.topk,
                                                static_smem[dev], device_sms(), bps[dev], tile);
    if (!q.ok || q.R > nr) return CSA2_ERR_UNSUPPORTED;
    if (cudaMemsetAsync(L.hist1, 0, L.sync_bytes, st) != cudaSuccess) return CSA2_ERR_CUDA;
    fd::Params p = base;
    p.R = (int32_t)q.R;
    p.row0 = row0;
    row0 += q.R;
    p.per_cta = q.per_cta;
    p.g_row = q.g_row;
    p.hist1 = L.hist1;
    p.arrive = L.arrive;
    p.cnt = L.cnt;
    p.cand = L.cand;
    p.part = L.part;
    p.off_sc = q.off_sc;
    p.off_hist = q.off_hist;
    p.off_qs = q.off_qs;
    p.cap = q.cap;
    p.stages = q.stages;
    p.p_att = q.P;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)q.G, 1, 1);
    cfg.blockDim = dim3(fd::kThreads, 1, 1);
    cfg.dynamicSmemBytes = q.dyn;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    TraceScope ts(p.do_attn ? "decode_fused" : "decode_fused_topk", st);
    if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return CSA2_ERR_CUDA;
  }
  return CSA2_OK;
}

using FusedRun = csa2_status (*)(const fd::Params &, int64_t, cudaStream_t, void *, size_t);

FusedRun pick_fused(int32_t d_I, int32_t H_I, int32_t D, bool fp4_keys) {
#define CSA2_FD_CASE(DI, HI, KF)                                                  \
  if (d_I == DI && H_I == HI)                                                     \
    return D == 128 ? &run_fused_t<DI, HI, 128, KF> : &run_fused_t<DI, HI, 64, KF>;
  if (fp4_keys) {
    CSA2_FD_CASE(32, 4, fd::kKeysFp4) CSA2_FD_CASE(64, 4, fd::kKeysFp4)
    return nullptr;
  }
  CSA2_FD_CASE(32, 4, fd::kKeysInt8) CSA2_FD_CASE(32, 8, fd::kKeysInt8)
  CSA2_FD_CASE(64, 4, fd::kKeysInt8) CSA2_FD_CASE(64, 8, fd::kKeysInt8)
#undef CSA2_FD_CASE
  return nullptr;
}

// Index + top-k (and, when `att` is given, the layer's attention fused into
// the same per-row cluster kernel), in passes of R rows.
// k_exps: NULL for int8 index keys; else the keys are FP4 (k_idx holds the
// codes) and only the fused decode kernel serves the call.
// A Full layer's candidate pool, kept from the same scan as its selection
// (decode rows): the best n_blocks blocks of `block` positions by their
// largest score, expanded to positions.  Scratch regions after the scan's.
struct PoolExt {
  uint32_t *bkey;   // [B, nb] block maxima as score keys (fused kernel)
  float *bscores;   // [B, round4(nb)] block maxima
  uint32_t *bhist;  // [B, kHistStride] their digit-1 histograms
  uint2 *bcand;     // [B, nb] candidate overflow of the block top-k
  int32_t *bidx;    // [B, n_blocks] kept blocks
  size_t bytes;
};
struct PoolReq {
  int32_t block, n_blocks;
  int32_t *pool;  // [B, n_blocks * block] output
  PoolExt X;
};
csa2_status pool_select_expand(const PoolExt &X, int64_t B, int64_t N, int32_t block,
                               int32_t n_blocks, int32_t *pool, cudaStream_t st);
csa2_status pool_from_block_keys(const PoolExt &X, int64_t B, int64_t N, int32_t block,
                                 int32_t n_blocks, int32_t *pool, cudaStream_t st);

// k_exps != nullptr: FP4 index keys (k_idx holds the codes); decode rows
// only.  pr != nullptr: also keep the rows' candidate pool (decode rows).
csa2_status run_index_topk(const int8_t *q_idx, const float *w, const int8_t *k_idx,
                           const uint8_t *k_exps, int32_t B, int32_t T, int32_t H_I, int32_t d_I,
                           int64_t N, int64_t n_prior, int32_t ratio, int32_t topk,
                           int32_t *idx_out, float *score_out, const AttnArgs *att, void *ws,
                           size_t ws_bytes, cudaStream_t st, const PoolReq *pr = nullptr) {
  const int64_t rows = int64_t(B) * T;
  const bool fp4 = k_exps != nullptr;
  const bool decode = T == 1 && n_prior < 0;
  if ((fp4 || pr) && !decode) return CSA2_ERR_UNSUPPORTED;
  if (fused_enabled() && score_out == nullptr &&
      fused_shape_ok(T, H_I, d_I, N, n_prior, topk, fp4) &&
      (!att || (att->H <= fd::kHeads && (att->D == 64 || att->D == 128)))) {
    const FusedRun run = pick_fused(d_I, H_I, att ? att->D : 64, fp4);
    if (run) {
      fd::Params p{};
      p.q_idx = q_idx;
      p.w = w;
      p.k_idx = k_idx;
      p.k_exps = k_exps;
      if (pr) {
        const int64_t nb = ceil_div(N, pr->block);
        if (cudaMemsetAsync(pr->X.bkey, 0, size_t(B) * nb * 4, st) != cudaSuccess)
          return CSA2_ERR_CUDA;
        p.bkey = pr->X.bkey;
        p.pool_block = pr->block;
        p.n_pool_blocks = nb;
      }
      p.N = N;
      p.topk = topk;
      p.idx = idx_out;
      if (att) {
        p.do_attn = 1;
        p.q = att->q;
        p.codes = att->codes;
        p.scales = att->scales;
        p.win_k = att->win_k;
        p.win_v = att->win_v;
        p.H = att->H;
        p.W = att->W;
        p.q_scale = att->sm_scale * 1.4426950408889634f;
        p.out = att->out;
        p.lse = att->lse;
      }
      csa2_status rc = run(p, rows, st, ws, ws_bytes);
      if (rc == CSA2_OK && pr)
        rc = pool_from_block_keys(pr->X, B, N, pr->block, pr->n_blocks, pr->pool, st);
      if (rc != CSA2_ERR_UNSUPPORTED) return rc;  // else the general path below
    }
  }
  if (!fp4 && !pr && pf_eligible(T, H_I, d_I, N, topk, score_out)) {
    const int64_t Rp = pf_rows_per_pass(T, N, d_I);
    const PfWs Lp0 = pf_ws_layout(nullptr, Rp, N, d_I);
    if (!ws || ws_bytes < Lp0.bytes || !aligned(ws, 16)) return CSA2_ERR_WORKSPACE;
    const PfRun run = pick_pf(d_I, H_I);
    if (!run) return CSA2_ERR_UNSUPPORTED;
    const PfWs Lp = pf_ws_layout(ws, Rp, N, d_I);
    if (run(q_idx, w, k_idx, B, T, N, n_prior, ratio, topk, idx_out, Lp, Rp, st) != CSA2_OK)
      return CSA2_ERR_CUDA;
    if (!att) return CSA2_OK;
    return run_attn(att->q, att->codes, att->scales, idx_out, att->win_k, att->win_v, B, T,
                    att->H, att->D, N, topk, att->W, att->sm_scale, att->out, att->lse, st);
  }
  const int64_t R0 = topk_rows_per_pass(rows, N);
  const TopkWs L0 = topk_ws_layout(nullptr, R0, N);
  if (!ws || ws_bytes < L0.bytes || !aligned(ws, 16)) return CSA2_ERR_WORKSPACE;
  const TopkWs L = topk_ws_layout(ws, R0, N);
  const ScanLaunch scan = fp4 ? nullptr : pick_scan(d_I, H_I);
  const ScanLaunchFp4 scan4 = fp4 ? pick_scan_fp4(d_I, H_I) : nullptr;
  if (!scan && !scan4) return CSA2_ERR_UNSUPPORTED;
  if (fp4 && N % 16 != 0) return CSA2_ERR_UNSUPPORTED;
  // several rows per sequence: whole sequences per pass, one shared scan each
  const ScanLaunch scan_group = fp4 ? nullptr : pick_scan_group(d_I, H_I, T);
  const int64_t R = (scan_group && R0 >= T) ? R0 / T * T : R0;
  const int sms = device_sms();
  const int64_t nbk = pr ? ceil_div(N, pr->block) : 0;
  const int64_t bstride = (nbk + 3) & ~int64_t(3);
  // the scan takes the block maxima itself for blocks of 2^i <= 16 positions
  const ScanLaunchBM scan_bm =
      (pr && !fp4 && T == 1 && score_out == nullptr && pr->block <= 16 &&
       (pr->block & (pr->block - 1)) == 0)
          ? pick_scan_bm(d_I, H_I)
          : nullptr;
  if (pr && cudaMemsetAsync(pr->X.bhist, 0, size_t(B) * kHistStride * 4, st) != cudaSuccess)
    return CSA2_ERR_CUDA;
  // Attention after the selection.  With many rows per launch (8 or fewer
  // selecting CTAs per row) a separate kernel fed by each selecting CTA's
  // list, its CTAs' partials merged by the row's last CTA (a few partials
  // per row), when the workspace holds the lists (layer calls size it so);
  // with few rows (16 CTAs per row) the per-row cluster kernel attends
  // itself and merges its 16 partials on chip.
  const bool handoff_ok =
      att && topk <= kSelCap && att->H > 0 &&
      ws_bytes >= L0.bytes + handoff_layout(nullptr, R0, topk, att->H, att->D).bytes;
  const HandoffWs Hw = handoff_ok ? handoff_layout(static_cast<char *>(ws) + L0.bytes, R0, topk,
                                                   att->H, att->D)
                                  : HandoffWs{};

  for (int64_t row0 = 0; row0 < rows; row0 += R) {
    const int64_t nr = std::min<int64_t>(R, rows - row0);
    if (cudaMemsetAsync(L.hist1, 0, size_t(nr) * kHistStride * 4, st) != cudaSuccess)
      return CSA2_ERR_CUDA;
    const int64_t stride = score_out ? N : score_stride(N);
    float *scores = score_out ? score_out + row0 * N : L.scores;
    // scan: about two CTAs per SM in total (the slices of a row are balanced
    // to 16 keys), at least 256 keys per CTA
    const bool grouped = scan_group && R >= T;  // passes hold whole sequences
    const int64_t units = grouped ? nr / T : nr;  // CTA groups: sequences or rows
    const int64_t g_want = std::max<int64_t>(1, (2 * sms + units / 2) / units);
    const int64_t g_max = std::max<int64_t>(1, N / 256);
    const int G = (int)std::min(g_want, g_max);
    {
      TraceScope ts("index_scan", st);
      if (scan_bm)  // a Full row's pool: the block maxima come with the scores
        scan_bm(dim3(G, (unsigned)units), st, q_idx, w, k_idx, N, row0, scores, stride, L.hist1,
                ScanBlockMax{pr->X.bscores + row0 * bstride, bstride,
                             pr->X.bhist + row0 * kHistStride, pr->block});
      else if (scan4)
        scan4(dim3(G, (unsigned)units), st, q_idx, w, k_idx, k_exps, T, N, n_prior, ratio, row0,
              scores, stride, L.hist1, score_out != nullptr);
      else
        (grouped ? scan_group : scan)(dim3(G, (unsigned)units), st, q_idx, w, k_idx, T, N,
                                      n_prior, ratio, row0, scores, stride, L.hist1,
                                      score_out != nullptr);
    }
    if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
    RowParams p{};
    p.scores = scores;
    p.score_stride = stride;
    p.hist1 = L.hist1;
    p.cand = L.cand;
    p.N = N;
    p.T = T;
    p.n_prior = n_prior;
    p.ratio = ratio;
    p.row0 = row0;
    p.topk = topk;
    p.idx = idx_out;
    p.do_topk = 1;
    int D = 64;
    const bool handoff = handoff_ok && row_cluster_size(nr, att->D) <= 8;
    if (att) {
      p.codes = att->codes;
      p.scales = att->scales;
      D = att->D;
      if (handoff) {  // each CTA's selection goes to the attention kernel
        p.lists = Hw.lists;
        p.list_stride = topk;
      } else {  // attention in the same kernel
        p.q = att->q;
        p.win_k = att->win_k;
        p.win_v = att->win_v;
        p.H = att->H;
        p.W = att->W;
        p.q_scale = att->sm_scale * 1.4426950408889634f;
        p.out = att->out;
        p.lse = att->lse;
        p.do_attn = 1;
      }
    }
    if (launch_row(p, D, nr, st) != CSA2_OK) return CSA2_ERR_CUDA;
    if (handoff) {  // the attention of these rows, overlapping the selection
      ah::Params hp{};
      hp.a.q = att->q;
      hp.a.codes = att->codes;
      hp.a.scales = att->scales;
      hp.a.win_k = att->win_k;
      hp.a.win_v = att->win_v;
      hp.a.N = N;
      hp.a.T = T;
      hp.a.H = att->H;
      hp.a.W = att->W;
      hp.a.topk = topk;
      hp.a.q_scale = att->sm_scale * 1.4426950408889634f;
      hp.a.out = att->out;
      hp.a.lse = att->lse;
      hp.a.row0 = row0;
      hp.lists = Hw.lists;
      hp.list_stride = topk;
      hp.flags = L.hist1 + kBins1;
      hp.flag_stride = kHistStride;
      hp.part = Hw.part;
      hp.G = row_cluster_size(nr, D);
      if (launch_attn_handoff(hp, D, nr, st) != CSA2_OK) return CSA2_ERR_CUDA;
    }
    if (pr && !scan_bm) {  // block maxima of these rows' scores, before the next pass reuses them
      TraceScope ts("pool_block_max", st);
      block_max_kernel<<<dim3((unsigned)ceil_div(nbk, kPoolThreads), (unsigned)nr), kPoolThreads,
                         0, st>>>(scores, stride, N, pr->block, pr->X.bscores + row0 * bstride,
                                  bstride, pr->X.bhist + row0 * kHistStride);
      if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
    }
  }
  if (pr) return pool_select_expand(pr->X, B, N, pr->block, pr->n_blocks, pr->pool, st);
  return CSA2_OK;
}

// ---------------------------------------------------------------------------
// Hierarchical indexer (pool.cuh): the pool of a Full row, the top-k of a
// Reindex row within a pool.  Decode shape: one query per sequence.
// ---------------------------------------------------------------------------
constexpr int32_t kPoolMaxBlock = 64;
constexpr int64_t kPoolMaxLen = 65536;

struct PoolWs {
  TopkWs t;         // full-row scores, their histograms, candidate overflow
  float *bscores;   // [R, round4(nb)] block maxima
  uint32_t *bhist;  // [R, kHistStride] their digit-1 histograms
  int32_t *bidx;    // [B, n_blocks] kept blocks
  size_t bytes;
};

PoolWs pool_ws_layout(void *base, int64_t R, int64_t B, int64_t N, int32_t block,
                      int32_t n_blocks) {
  PoolWs w{};
  w.t = topk_ws_layout(base, R, N);
  size_t off = w.t.bytes;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  const int64_t nb = ceil_div(N, block);
  const size_t o_bs = take(size_t(R) * size_t((nb + 3) & ~int64_t(3)) * 4);
  const size_t o_bh = take(size_t(R) * kHistStride * 4);
  const size_t o_bi = take(size_t(B) * n_blocks * 4);
  char *p = static_cast<char *>(base);
  w.bscores = reinterpret_cast<float *>(p + o_bs);
  w.bhist = reinterpret_cast<uint32_t *>(p + o_bh);
  w.bidx = reinterpret_cast<int32_t *>(p + o_bi);
  w.bytes = off;
  return w;
}

struct PoolTopkWs {
  TopkWs t;     // pool scores, their histograms, candidate overflow
  int32_t *sel; // [B, topk] selected pool slots
  size_t bytes;
};

PoolTopkWs pool_topk_ws_layout(void *base, int64_t R, int64_t B, int64_t P, int32_t topk) {
  PoolTopkWs w{};
  w.t = topk_ws_layout(base, R, P);
  const size_t o = w.t.bytes;
  w.sel = reinterpret_cast<int32_t *>(static_cast<char *>(base) + o);
  w.bytes = o + align_up(size_t(B) * topk * 4, 256);
  return w;
}

csa2_status check_pool_common(const int8_t *q_idx, const float *w, const int8_t *k_idx,
                              int32_t B, int32_t H_I, int32_t d_I, int64_t N) {
  if (B < 0 || N < 0 || H_I < 1 || d_I < 1 || d_I % 16 != 0) return CSA2_ERR_INVALID_ARG;
  if (!scan_shape_supported(H_I, d_I) || N >= (int64_t(1) << 31) - 1 || B > 65535)
    return CSA2_ERR_UNSUPPORTED;
  if (B == 0) return CSA2_OK;
  if (!q_idx || !w || (N > 0 && !k_idx)) return CSA2_ERR_INVALID_ARG;
  if (!aligned(q_idx, 16) || (k_idx && !aligned(k_idx, 16)) || !aligned(w, 4))
    return CSA2_ERR_INVALID_ARG;
  return CSA2_OK;
}

csa2_status run_index_pool(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B,
                           int32_t H_I, int32_t d_I, int64_t N, int32_t block, int32_t n_blocks,
                           int32_t *pool_out, void *ws, size_t ws_bytes, cudaStream_t st) {
  const int64_t P = int64_t(n_blocks) * block;
  if (N == 0) {  // nothing stored: an empty pool
    return cudaMemsetAsync(pool_out, 0xff, size_t(B) * P * 4, st) == cudaSuccess ? CSA2_OK
                                                                                : CSA2_ERR_CUDA;
  }
  const int64_t rows = B;
  const int64_t R = topk_rows_per_pass(rows, N);
  const PoolWs L0 = pool_ws_layout(nullptr, R, B, N, block, n_blocks);
  if (!ws || ws_bytes < L0.bytes || !aligned(ws, 16)) return CSA2_ERR_WORKSPACE;
  const PoolWs L = pool_ws_layout(ws, R, B, N, block, n_blocks);
  const ScanLaunch scan = pick_scan(d_I, H_I);
  if (!scan) return CSA2_ERR_UNSUPPORTED;
  const int sms = device_sms();
  const int64_t nb = ceil_div(N, block);
  const int64_t bstride = (nb + 3) & ~int64_t(3);
  for (int64_t row0 = 0; row0 < rows; row0 += R) {
    const int64_t nr = std::min<int64_t>(R, rows - row0);
    // the Full row's scores over the whole store
    if (cudaMemsetAsync(L.t.hist1, 0, size_t(nr) * kHistStride * 4, st) != cudaSuccess)
      return CSA2_ERR_CUDA;
    const int64_t g_want = std::max<int64_t>(1, (2 * sms + nr / 2) / nr);
    const int G = (int)std::min(g_want, std::max<int64_t>(1, N / 256));
    {
      TraceScope ts("index_scan", st);
      scan(dim3(G, (unsigned)nr), st, q_idx, w, k_idx, 1, N, -1, 1, row0, L.t.scores,
           score_stride(N), L.t.hist1, 0);
    }
    if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
    // block maxima and their histogram
    if (cudaMemsetAsync(L.bhist, 0, size_t(nr) * kHistStride * 4, st) != cudaSuccess)
      return CSA2_ERR_CUDA;
    {
      TraceScope ts("pool_block_max", st);
      block_max_kernel<<<dim3((unsigned)ceil_div(nb, kPoolThreads), (unsigned)nr), kPoolThreads,
                         0, st>>>(L.t.scores, score_stride(N), N, block, L.bscores, bstride,
                                  L.bhist);
    }
    if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
    // the best n_blocks blocks, ascending
    RowParams p{};
    p.scores = L.bscores;
    p.score_stride = bstride;
    p.hist1 = L.bhist;
    p.cand = L.t.cand;
    p.N = nb;
    p.T = 1;
    p.n_prior = -1;
    p.ratio = 1;
    p.row0 = row0;
    p.topk = n_blocks;
    p.idx = L.bidx;
    p.do_topk = 1;
    if (launch_row(p, 64, nr, st) != CSA2_OK) return CSA2_ERR_CUDA;
  }
  {
    TraceScope ts("pool_expand", st);
    expand_pool_kernel<<<dim3((unsigned)ceil_div(P, kPoolThreads), (unsigned)B), kPoolThreads, 0,
                         st>>>(L.bidx, n_blocks, block, N, pool_out);
  }
  return after_launch();
}

csa2_status run_pool_topk(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B,
                          int32_t H_I, int32_t d_I, int64_t N, const int32_t *pool, int32_t P,
                          int32_t topk, int32_t *idx_out, void *ws, size_t ws_bytes,
                          cudaStream_t st) {
  if (P == 0) {  // an empty pool selects nothing
    return cudaMemsetAsync(idx_out, 0xff, size_t(B) * topk * 4, st) == cudaSuccess
               ? CSA2_OK
               : CSA2_ERR_CUDA;
  }
  const int64_t rows = B;
  const int64_t R = topk_rows_per_pass(rows, P);
  const PoolTopkWs L0 = pool_topk_ws_layout(nullptr, R, B, P, topk);
  if (!ws || ws_bytes < L0.bytes || !aligned(ws, 16)) return CSA2_ERR_WORKSPACE;
  const PoolTopkWs L = pool_topk_ws_layout(ws, R, B, P, topk);
  const int64_t pstride = score_stride(P);
  for (int64_t row0 = 0; row0 < rows; row0 += R) {
    const int64_t nr = std::min<int64_t>(R, rows - row0);
    if (cudaMemsetAsync(L.t.hist1, 0, size_t(nr) * kHistStride * 4, st) != cudaSuccess)
      return CSA2_ERR_CUDA;
    {
      TraceScope ts("pool_scan", st);
      pool_scan_kernel<<<dim3((unsigned)ceil_div(P, kPoolThreads), (unsigned)nr), kPoolThreads, 0,
                         st>>>(q_idx + row0 * H_I * d_I, w + row0 * H_I,
                               N > 0 ? k_idx + row0 * N * d_I : k_idx, H_I, d_I, N,
                               pool + row0 * P, P, L.t.scores, pstride, L.t.hist1);
    }
    if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
    RowParams p{};
    p.scores = L.t.scores;
    p.score_stride = pstride;
    p.hist1 = L.t.hist1;
    p.cand = L.t.cand;
    p.N = P;
    p.T = 1;
    p.n_prior = -1;
    p.ratio = 1;
    p.row0 = row0;
    p.topk = topk;
    p.idx = L.sel;
    p.do_topk = 1;
    if (launch_row(p, 64, nr, st) != CSA2_OK) return CSA2_ERR_CUDA;
  }
  {
    TraceScope ts("pool_map", st);
    map_pool_kernel<<<dim3((unsigned)ceil_div(topk, kPoolThreads), (unsigned)B), kPoolThreads, 0,
                      st>>>(L.sel, topk, pool, P, N, idx_out);
  }
  return after_launch();
}

// ---------------------------------------------------------------------------
// Attention with given indices.
// ---------------------------------------------------------------------------
csa2_status check_attn_args(const uint16_t *q, const uint8_t *codes, const float *scales,
                            const int32_t *idx, const uint16_t *win_k, const uint16_t *win_v,
                            int32_t B, int32_t T, int32_t H, int32_t D, int64_t N, int32_t topk,
                            int32_t W, const float *out, const float *lse) {
  if (B < 0 || T < 0 || H < 1 || D < 1 || N < 0 || topk < 0 || W < 0) return CSA2_ERR_INVALID_ARG;
  if (D % 16 != 0) return CSA2_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || H > 128 || topk > 65536 || W > 4096 ||
      N >= (int64_t(1) << 31) - 1)
    return CSA2_ERR_UNSUPPORTED;
  if (int64_t(B) * T == 0) return CSA2_OK;
  if (!q || !out || (topk > 0 && !idx) || (topk > 0 && N > 0 && (!codes || !scales)) ||
      (W > 0 && (!win_k || !win_v)))
    return CSA2_ERR_INVALID_ARG;
  if (!aligned(q, 16) || (codes && !aligned(codes, 16)) || (scales && !aligned(scales, 16)) ||
      (idx && !aligned(idx, 4)) || (win_k && !aligned(win_k, 16)) ||
      (win_v && !aligned(win_v, 16)) || !aligned(out, 16) || (lse && !aligned(lse, 4)))
    return CSA2_ERR_INVALID_ARG;
  return CSA2_OK;
}

constexpr int64_t kAttnRowsPerLaunch = 16384;

// Many rows: one CTA per (row, 16-head pass), every SM busy with whole rows.
template <int D>
csa2_status launch_attn_rows(const ar::Params &p, int64_t nr, cudaStream_t st) {
  const size_t smem = sizeof(ar::Smem<D>);
  static std::atomic<bool> done[256];  // per device: attributes set
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 256 || !done[dev].load(std::memory_order_acquire)) {
    if (set_smem_attr(ar::attn_rows_kernel<D>, smem, false) != CSA2_OK) return CSA2_ERR_CUDA;
    if (dev >= 0 && dev < 256) done[dev].store(true, std::memory_order_release);
  }
  TraceScope ts("attend_rows", st);
  const unsigned passes = (unsigned)ceil_div(p.H, ar::kHeads);
  ar::attn_rows_kernel<D><<<dim3((unsigned)nr, passes), ar::kThreads, smem, st>>>(p);
  return after_launch();
}

// Rows at which the per-row CTA kernel takes over from the cluster kernel
// (which spreads one row over up to 16 SMs: better while rows are few).
inline int64_t attn_rows_threshold() { return 2 * int64_t(device_sms()); }

csa2_status run_attn(const uint16_t *q, const uint8_t *codes, const float *scales,
                     const int32_t *idx, const uint16_t *win_k, const uint16_t *win_v, int32_t B,
                     int32_t T, int32_t H, int32_t D, int64_t N, int32_t topk, int32_t W,
                     float sm_scale, float *out, float *lse, cudaStream_t st) {
  const int64_t rows = int64_t(B) * T;
  if (rows >= attn_rows_threshold()) {
    ar::Params a{};
    a.q = q;
    a.codes = codes;
    a.scales = scales;
    a.idx = idx;
    a.win_k = win_k;
    a.win_v = win_v;
    a.N = N;
    a.T = T;
    a.H = H;
    a.W = W;
    a.topk = topk;
    a.q_scale = sm_scale * 1.4426950408889634f;
    a.out = out;
    a.lse = lse;
    for (int64_t row0 = 0; row0 < rows; row0 += kAttnRowsPerLaunch) {
      const int64_t nr = std::min<int64_t>(kAttnRowsPerLaunch, rows - row0);
      a.row0 = row0;
      const csa2_status rc =
          D == 128 ? launch_attn_rows<128>(a, nr, st) : launch_attn_rows<64>(a, nr, st);
      if (rc != CSA2_OK) return rc;
    }
    return CSA2_OK;
  }
  ar::Params a{};
  a.q = q;
  a.codes = codes;
  a.scales = scales;
  a.idx = idx;
  a.win_k = win_k;
  a.win_v = win_v;
  a.N = N;
  a.T = T;
  a.H = H;
  a.W = W;
  a.topk = topk;
  a.q_scale = sm_scale * 1.4426950408889634f;
  a.out = out;
  a.lse = lse;
  for (int64_t row0 = 0; row0 < rows; row0 += kAttnRowsPerLaunch) {
    const int64_t nr = std::min<int64_t>(kAttnRowsPerLaunch, rows - row0);
    a.row0 = row0;
    if (launch_attn_cluster(a, D, nr, false, st) != CSA2_OK) return CSA2_ERR_CUDA;
  }
  return CSA2_OK;
}

// ---------------------------------------------------------------------------
// Candidate pools kept by Full layers for CSA2_REINDEX_POOL layers: block
// maxima of the Full rows' scores (from the scan's score rows, or left as
// score keys by the fused kernel), the best pool_blocks blocks by the row
// kernel's exact top-k, expanded to positions.  Scratch after the scan's.
// ---------------------------------------------------------------------------
bool pool_dims_ok(const csa2_dims *d) {
  return d->pool_block >= 1 && d->pool_block <= kPoolMaxBlock && d->pool_blocks >= 1 &&
         int64_t(d->pool_block) * d->pool_blocks <= kPoolMaxLen && d->T == 1 && d->n_prior < 0;
}

PoolExt pool_ext_layout(void *base, int64_t B, int64_t N, int32_t block, int32_t n_blocks) {
  PoolExt w{};
  const int64_t nb = ceil_div(N, block);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  const size_t o_k = take(size_t(B) * nb * 4);
  const size_t o_s = take(size_t(B) * ((nb + 3) & ~int64_t(3)) * 4);
  const size_t o_h = take(size_t(B) * kHistStride * 4);
  const size_t o_c = take(size_t(B) * nb * 8);
  const size_t o_i = take(size_t(B) * n_blocks * 4);
  char *p = static_cast<char *>(base);
  w.bkey = reinterpret_cast<uint32_t *>(p + o_k);
  w.bscores = reinterpret_cast<float *>(p + o_s);
  w.bhist = reinterpret_cast<uint32_t *>(p + o_h);
  w.bcand = reinterpret_cast<uint2 *>(p + o_c);
  w.bidx = reinterpret_cast<int32_t *>(p + o_i);
  w.bytes = off;
  return w;
}

// The pool regions start after the largest scan / fused-kernel workspace.
// Workspace of a layer's selection and its hand-off to the attention
// kernel (the top-k regions, then the lists and partials).
size_t handoff_ws_bytes(const csa2_dims *d) {
  const int64_t R = topk_rows_per_pass(int64_t(d->B) * d->T, d->N);
  return topk_ws_layout(nullptr, R, d->N).bytes +
         handoff_layout(nullptr, R, d->topk, d->H, d->D).bytes;
}

size_t pool_ext_offset(const csa2_dims *d) {
  return align_up(std::max(fused_ws_bytes(int64_t(d->B) * d->T, d->N),
                           handoff_ws_bytes(d)),
                  256);
}

// The best n_blocks blocks of each row (block scores and their digit-1
// histograms in X) -> the pool's positions.
csa2_status pool_select_expand(const PoolExt &X, int64_t B, int64_t N, int32_t block,
                               int32_t n_blocks, int32_t *pool, cudaStream_t st) {
  const int64_t nb = ceil_div(N, block);
  RowParams p{};
  p.scores = X.bscores;
  p.score_stride = (nb + 3) & ~int64_t(3);
  p.hist1 = X.bhist;
  p.cand = X.bcand;
  p.N = nb;
  p.T = 1;
  p.n_prior = -1;
  p.ratio = 1;
  p.row0 = 0;
  p.topk = n_blocks;
  p.idx = X.bidx;
  p.do_topk = 1;
  if (launch_row(p, 64, B, st) != CSA2_OK) return CSA2_ERR_CUDA;
  const int64_t P = int64_t(block) * n_blocks;
  TraceScope ts("pool_expand", st);
  expand_pool_kernel<<<dim3((unsigned)ceil_div(P, kPoolThreads), (unsigned)B), kPoolThreads, 0,
                       st>>>(X.bidx, n_blocks, block, N, pool);
  return after_launch();
}

// After the fused kernel: block maxima kept as keys -> block scores -> pool.
csa2_status pool_from_block_keys(const PoolExt &X, int64_t B, int64_t N, int32_t block,
                                 int32_t n_blocks, int32_t *pool, cudaStream_t st) {
  const int64_t nb = ceil_div(N, block);
  if (cudaMemsetAsync(X.bhist, 0, size_t(B) * kHistStride * 4, st) != cudaSuccess)
    return CSA2_ERR_CUDA;
  {
    TraceScope ts("pool_block_keys", st);
    block_keys_to_scores_kernel<<<dim3((unsigned)ceil_div(nb, kPoolThreads), (unsigned)B),
                                  kPoolThreads, 0, st>>>(X.bkey, nb, X.bscores,
                                                         (nb + 3) & ~int64_t(3), X.bhist);
    if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
  }
  return pool_select_expand(X, B, N, block, n_blocks, pool, st);
}

// ---------------------------------------------------------------------------
// Mode tables.
// ---------------------------------------------------------------------------
csa2_status check_modes(const csa2_layer_mode *m, int32_t L) {
  if (!m || L <= 0) return CSA2_ERR_INVALID_ARG;
  for (int32_t l = 0; l < L; ++l) {
    const int32_t mode = m[l].mode, kv = m[l].kv_src, ix = m[l].idx_src;
    switch (mode) {
      case CSA2_FULL:
        if (kv != l || ix != l) return CSA2_ERR_INVALID_ARG;
        break;
      case CSA2_REINDEX:
      case CSA2_REINDEX_POOL:
        if (kv < 0 || kv >= l || m[kv].mode != CSA2_FULL || ix != l) return CSA2_ERR_INVALID_ARG;
        break;
      case CSA2_REUSE:
        if (ix < 0 || ix >= l || m[ix].mode == CSA2_REUSE || kv != m[ix].kv_src)
          return CSA2_ERR_INVALID_ARG;
        break;
      default:
        return CSA2_ERR_INVALID_ARG;
    }
  }
  return CSA2_OK;
}

}  // namespace

// ===========================================================================
// Exported entry points.
// ===========================================================================
extern "C" {

const char *csa2_status_string(int32_t status) {
  switch (status) {
    case CSA2_OK: return "CSA2_OK";
    case CSA2_ERR_INVALID_ARG: return "CSA2_ERR_INVALID_ARG: invalid argument";
    case CSA2_ERR_UNSUPPORTED: return "CSA2_ERR_UNSUPPORTED: shape outside the compiled set";
    case CSA2_ERR_CUDA: return "CSA2_ERR_CUDA: CUDA launch or query failed";
    case CSA2_ERR_WORKSPACE: return "CSA2_ERR_WORKSPACE: workspace missing or too small";
    case CSA2_ERR_DEVICE_STATUS: return "CSA2_ERR_DEVICE_STATUS: a kernel recorded an error";
    default: return "unknown csa2 status";
  }
}

int32_t csa2_version(void) { return 10000; }

csa2_status csa2_pack_fp4(const float *src, int64_t rows, int32_t D, uint8_t *codes,
                          float *scales, void *stream) {
  if (rows < 0 || D <= 0 || D % 16 != 0) return CSA2_ERR_INVALID_ARG;
  if (rows == 0) return CSA2_OK;
  if (!src || !codes || !scales || !aligned(src, 16) || !aligned(codes, 8) || !aligned(scales, 4))
    return CSA2_ERR_INVALID_ARG;
  const int64_t groups = rows * (D / 16);
  const int64_t blocks = std::min<int64_t>(ceil_div(groups, 256), int64_t(device_sms()) * 16);
  TraceScope ts("pack_fp4", as_stream(stream));
  pack_fp4_kernel<<<(unsigned)blocks, 256, 0, as_stream(stream)>>>(src, groups, codes, scales);
  return after_launch();
}

namespace {
// Where the bytes [p, p + len) live: 0 = this device's memory, 1 = page-
// locked host memory the device addresses at the same pointer, -1 = neither
// (pageable host memory, another device's memory), checked at both ends.
csa2_status memory_kind(const void *p, int64_t len, int &kind) {
  kind = -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CSA2_ERR_CUDA;
  int k[2];
  const char *ends[2] = {static_cast<const char *>(p), static_cast<const char *>(p) + (len - 1)};
  for (int e = 0; e < 2; ++e) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, ends[e]) != cudaSuccess) {
      cudaGetLastError();
      return CSA2_ERR_CUDA;
    }
    if ((a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && a.device == dev)
      k[e] = 0;
    else if (a.type == cudaMemoryTypeHost && a.devicePointer == ends[e])
      k[e] = 1;
    else
      k[e] = -1;
  }
  if (k[0] == k[1]) kind = k[0];
  return CSA2_OK;
}
}  // namespace

csa2_status csa2_stage_copies(const csa2_copy2d *copies, int32_t n, void *stream) {
  if (n < 0 || n > kStageMax || (n > 0 && !copies)) return CSA2_ERR_INVALID_ARG;
  // every copy's sizes and alignment first, then where its memory lives
  for (int i = 0; i < n; ++i) {
    const csa2_copy2d &c = copies[i];
    if (c.rows < 0 || c.row_bytes < 0) return CSA2_ERR_INVALID_ARG;
    if (c.rows == 0 || c.row_bytes == 0) continue;
    if (!c.src || !c.dst || !aligned(c.src, 16) || !aligned(c.dst, 16) || c.row_bytes % 16 != 0 ||
        c.src_stride < 0 || c.src_stride % 16 != 0 || c.dst_stride % 16 != 0 ||
        (c.rows > 1 && c.dst_stride < c.row_bytes))
      return CSA2_ERR_INVALID_ARG;
  }
  StageList L{};
  int64_t most = 0;
  int m = 0;
  for (int i = 0; i < n; ++i) {
    const csa2_copy2d &c = copies[i];
    if (c.rows == 0 || c.row_bytes == 0) continue;
    int ks, kd;
    csa2_status rc = memory_kind(c.src, (c.rows - 1) * c.src_stride + c.row_bytes, ks);
    if (rc != CSA2_OK) return rc;
    rc = memory_kind(c.dst, (c.rows - 1) * c.dst_stride + c.row_bytes, kd);
    if (rc != CSA2_OK) return rc;
    if (ks < 0 || kd < 0) return CSA2_ERR_INVALID_ARG;
    L.c[m] = StageCopy{static_cast<const int4 *>(c.src), static_cast<int4 *>(c.dst), c.rows,
                       c.row_bytes / 16, c.src_stride / 16, c.dst_stride / 16, ks, kd};
    most = std::max(most, c.rows * (c.row_bytes / 16));
    ++m;
  }
  if (m == 0) return CSA2_OK;
  L.n = m;
  const int64_t x = std::min<int64_t>(ceil_div(most, int64_t(kStageThreads) * kStageUnroll),
                                      int64_t(device_sms()) * 4);
  TraceScope ts("stage_copies", as_stream(stream));
  stage_copies_kernel<<<dim3((unsigned)x, (unsigned)m), kStageThreads, 0, as_stream(stream)>>>(L);
  return after_launch();
}

csa2_status csa2_append_entry(const float *src, const int8_t *key, const int64_t *pos, int32_t B,
                              int32_t D, int32_t d_I, int64_t N, uint8_t *codes, float *scales,
                              int8_t *k_idx, void *stream) {
  if (B < 0 || D <= 0 || D % 16 != 0 || d_I <= 0 || d_I % 16 != 0 || N < 0)
    return CSA2_ERR_INVALID_ARG;
  if (B == 0) return CSA2_OK;
  if (!src || !key || !pos || (N > 0 && (!codes || !scales || !k_idx)) || !aligned(src, 16) ||
      !aligned(key, 16) || !aligned(pos, 8) || (codes && !aligned(codes, 8)) ||
      (scales && !aligned(scales, 4)) || (k_idx && !aligned(k_idx, 16)))
    return CSA2_ERR_INVALID_ARG;
  const int64_t units = int64_t(B) * (D / 16 + d_I / 16);
  const int64_t blocks = std::min<int64_t>(ceil_div(units, 128), int64_t(device_sms()) * 8);
  TraceScope ts("append_entry", as_stream(stream));
  append_entry_kernel<<<(unsigned)blocks, 128, 0, as_stream(stream)>>>(src, key, pos, B, D, d_I,
                                                                      N, codes, scales, k_idx);
  return after_launch();
}

csa2_status csa2_unpack_fp4(const uint8_t *codes, const float *scales, int64_t rows, int32_t D,
                            float *out, void *stream) {
  if (rows < 0 || D <= 0 || D % 16 != 0) return CSA2_ERR_INVALID_ARG;
  if (rows == 0) return CSA2_OK;
  if (!codes || !scales || !out || !aligned(codes, 8) || !aligned(scales, 4) || !aligned(out, 16))
    return CSA2_ERR_INVALID_ARG;
  const int64_t groups = rows * (D / 16);
  const int64_t blocks = std::min<int64_t>(ceil_div(groups, 256), int64_t(device_sms()) * 16);
  TraceScope ts("unpack_fp4", as_stream(stream));
  unpack_fp4_kernel<<<(unsigned)blocks, 256, 0, as_stream(stream)>>>(codes, scales, groups, out);
  return after_launch();
}

size_t csa2_index_topk_workspace_size(int32_t B, int32_t T, int32_t H_I, int32_t d_I, int64_t N,
                                      int32_t topk) {
  if (B < 0 || T < 0 || N < 0 || topk < 1 || !scan_shape_supported(H_I, d_I)) return 0;
  size_t bytes = topk_ws_bytes(B, T, N);
  if (pf_shape_ok(T, H_I, d_I, N, topk)) bytes = std::max(bytes, pf_ws_bytes(T, N, d_I));
  if (fused_shape_ok(T, H_I, d_I, N, -1, topk))
    bytes = std::max(bytes, fused_ws_bytes(int64_t(B) * T, N));
  return bytes;
}

csa2_status csa2_index_topk(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B,
                            int32_t T, int32_t H_I, int32_t d_I, int64_t N, int64_t n_prior,
                            int32_t ratio, int32_t topk, int32_t *idx_out, float *score_out,
                            void *ws, size_t ws_bytes, void *stream) {
  csa2_status rc = check_topk_args(q_idx, w, k_idx, B, T, H_I, d_I, N, n_prior, ratio, topk,
                                   idx_out, score_out);
  if (rc != CSA2_OK || int64_t(B) * T == 0) return rc;
  return run_index_topk(q_idx, w, k_idx, nullptr, B, T, H_I, d_I, N, n_prior, ratio, topk,
                        idx_out, score_out, nullptr, ws, ws_bytes, as_stream(stream));
}

csa2_status csa2_pack_index_keys_fp4(const float *src, int64_t rows, int32_t d_I,
                                     uint8_t *codes, uint8_t *exps, void *stream) {
  if (rows < 0 || d_I <= 0 || d_I % 32 != 0) return CSA2_ERR_INVALID_ARG;
  if (rows == 0) return CSA2_OK;
  if (!src || !codes || !exps || !aligned(src, 16) || !aligned(codes, 16))
    return CSA2_ERR_INVALID_ARG;
  const int64_t blocks = rows * (d_I / 32);
  const int64_t grid = std::min<int64_t>(ceil_div(blocks, 256), int64_t(device_sms()) * 16);
  TraceScope ts("pack_keys_fp4", as_stream(stream));
  pack_keys_fp4_kernel<<<(unsigned)grid, 256, 0, as_stream(stream)>>>(src, blocks, codes, exps);
  return after_launch();
}

size_t csa2_index_topk_fp4k_workspace_size(int32_t B, int32_t H_I, int32_t d_I, int64_t N,
                                           int32_t topk) {
  if (B < 0 || topk < 1 || topk > 65536 || !fp4_shape_ok(1, H_I, d_I, N, -1)) return 0;
  return std::max(fused_ws_bytes(B, N), topk_ws_bytes(B, 1, N));
}

csa2_status csa2_index_topk_fp4k(const int8_t *q_idx, const float *w, const uint8_t *k_codes,
                                 const uint8_t *k_exps, int32_t B, int32_t H_I, int32_t d_I,
                                 int64_t N, int32_t topk, int32_t *idx_out, void *ws,
                                 size_t ws_bytes, void *stream) {
  if (B < 0 || N < 0 || topk < 1 || H_I < 1 || d_I < 1 || d_I % 32 != 0)
    return CSA2_ERR_INVALID_ARG;
  if (topk > 65536 || !fp4_shape_ok(1, H_I, d_I, N, -1)) return CSA2_ERR_UNSUPPORTED;
  if (B == 0) return CSA2_OK;
  if (!q_idx || !w || !k_codes || !k_exps || !idx_out || !aligned(q_idx, 16) ||
      !aligned(k_codes, 16) || !aligned(k_exps, 16) || !aligned(w, 4) || !aligned(idx_out, 4))
    return CSA2_ERR_INVALID_ARG;
  return run_index_topk(q_idx, w, reinterpret_cast<const int8_t *>(k_codes), k_exps, B, 1, H_I,
                        d_I, N, -1, 4, topk, idx_out, nullptr, nullptr, ws, ws_bytes,
                        as_stream(stream));
}

size_t csa2_index_pool_workspace_size(int32_t B, int32_t H_I, int32_t d_I, int64_t N,
                                      int32_t block, int32_t n_blocks) {
  if (B < 0 || N < 0 || block < 1 || block > kPoolMaxBlock || n_blocks < 1 ||
      int64_t(n_blocks) * block > kPoolMaxLen || !scan_shape_supported(H_I, d_I))
    return 0;
  const int64_t R = topk_rows_per_pass(B, N);
  return pool_ws_layout(nullptr, R, B, N, block, n_blocks).bytes;
}

csa2_status csa2_index_pool(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B,
                            int32_t H_I, int32_t d_I, int64_t N, int32_t block, int32_t n_blocks,
                            int32_t *pool_out, void *ws, size_t ws_bytes, void *stream) {
  if (block < 1 || n_blocks < 1) return CSA2_ERR_INVALID_ARG;
  if (block > kPoolMaxBlock || int64_t(n_blocks) * block > kPoolMaxLen)
    return CSA2_ERR_UNSUPPORTED;
  csa2_status rc = check_pool_common(q_idx, w, k_idx, B, H_I, d_I, N);
  if (rc != CSA2_OK || B == 0) return rc;
  if (!pool_out || !aligned(pool_out, 4)) return CSA2_ERR_INVALID_ARG;
  return run_index_pool(q_idx, w, k_idx, B, H_I, d_I, N, block, n_blocks, pool_out, ws, ws_bytes,
                        as_stream(stream));
}

size_t csa2_pool_topk_workspace_size(int32_t B, int32_t P, int32_t topk) {
  if (B < 0 || P < 0 || P > kPoolMaxLen || topk < 1 || topk > 65536) return 0;
  const int64_t R = topk_rows_per_pass(B, P);
  return pool_topk_ws_layout(nullptr, R, B, P, topk).bytes;
}

csa2_status csa2_pool_topk(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B,
                           int32_t H_I, int32_t d_I, int64_t N, const int32_t *pool, int32_t P,
                           int32_t topk, int32_t *idx_out, void *ws, size_t ws_bytes,
                           void *stream) {
  if (P < 0 || topk < 1) return CSA2_ERR_INVALID_ARG;
  if (P > kPoolMaxLen || topk > 65536) return CSA2_ERR_UNSUPPORTED;
  csa2_status rc = check_pool_common(q_idx, w, k_idx, B, H_I, d_I, N);
  if (rc != CSA2_OK || B == 0) return rc;
  if (!idx_out || !aligned(idx_out, 4) || (P > 0 && (!pool || !aligned(pool, 4))))
    return CSA2_ERR_INVALID_ARG;
  return run_pool_topk(q_idx, w, k_idx, B, H_I, d_I, N, pool, P, topk, idx_out, ws, ws_bytes,
                       as_stream(stream));
}

size_t csa2_sparse_attn_workspace_size(int32_t B, int32_t T, int32_t H, int32_t D, int32_t topk,
                                       int32_t W) {
  (void)B;
  (void)T;
  (void)H;
  (void)D;
  (void)topk;
  (void)W;
  return 0;  // partial softmax states are merged on chip
}

csa2_status csa2_sparse_attn_decode(const uint16_t *q, const uint8_t *codes, const float *scales,
                                    const int32_t *idx, const uint16_t *win_k,
                                    const uint16_t *win_v, int32_t B, int32_t H, int32_t D,
                                    int64_t N, int32_t topk, int32_t W, float sm_scale, float *out,
                                    float *lse, void *ws, size_t ws_bytes, void *stream) {
  (void)ws;
  (void)ws_bytes;
  csa2_status rc = check_attn_args(q, codes, scales, idx, win_k, win_v, B, 1, H, D, N, topk, W,
                                   out, lse);
  if (rc != CSA2_OK || B == 0) return rc;
  return run_attn(q, codes, scales, idx, win_k, win_v, B, 1, H, D, N, topk, W, sm_scale, out, lse,
                  as_stream(stream));
}

csa2_status csa2_sparse_attn_prefill(const uint16_t *q, const uint8_t *codes, const float *scales,
                                     const int32_t *idx, const uint16_t *win_k,
                                     const uint16_t *win_v, int32_t B, int32_t T, int32_t H,
                                     int32_t D, int64_t N, int32_t topk, int32_t W,
                                     float sm_scale, float *out, float *lse, void *ws,
                                     size_t ws_bytes, void *stream) {
  (void)ws;
  (void)ws_bytes;
  csa2_status rc = check_attn_args(q, codes, scales, idx, win_k, win_v, B, T, H, D, N, topk, W,
                                   out, lse);
  if (rc != CSA2_OK || int64_t(B) * T == 0) return rc;
  return run_attn(q, codes, scales, idx, win_k, win_v, B, T, H, D, N, topk, W, sm_scale, out, lse,
                  as_stream(stream));
}

csa2_status csa2_validate_modes(const csa2_layer_mode *modes, int32_t L) {
  return check_modes(modes, L);
}

csa2_status csa2_group_cache_bytes(const csa2_layer_mode *modes, int32_t L, int64_t entries,
                                   int64_t numbers_per_entry, int64_t bits_per_number,
                                   uint64_t *bytes_out) {
  if (!bytes_out || entries < 0 || numbers_per_entry < 0 || bits_per_number <= 0)
    return CSA2_ERR_INVALID_ARG;
  csa2_status rc = check_modes(modes, L);
  if (rc != CSA2_OK) return rc;
  uint64_t stored = 0;
  for (int32_t l = 0; l < L; ++l) stored += (modes[l].mode == CSA2_FULL) ? 1u : 0u;
  const uint64_t bits = uint64_t(entries) * uint64_t(numbers_per_entry) * stored *
                        uint64_t(bits_per_number);
  *bytes_out = bits / 8u;
  return CSA2_OK;
}

size_t csa2_layer_group_workspace_size(const csa2_dims *d) {
  if (!d) return 0;
  if (d->B < 0 || d->T < 0 || d->H < 1 || (d->D != 64 && d->D != 128) || d->W < 0) return 0;
  size_t bytes = csa2_index_topk_workspace_size(d->B, d->T, d->H_I, d->d_I, d->N, d->topk);
  if (bytes) bytes = std::max(bytes, handoff_ws_bytes(d));
  if (bytes && (d->pool_block || d->pool_blocks)) {
    if (!pool_dims_ok(d)) return 0;
    bytes = std::max(bytes, pool_ext_offset(d) + pool_ext_layout(nullptr, d->B, d->N,
                                                                  d->pool_block,
                                                                  d->pool_blocks).bytes);
    const int64_t P = int64_t(d->pool_block) * d->pool_blocks;
    bytes = std::max(bytes, pool_topk_ws_layout(nullptr, topk_rows_per_pass(d->B, P), d->B, P,
                                                d->topk).bytes);
  }
  return bytes;
}

}  // extern "C"

namespace {

// Validate the table and the pointers of the layers in [l0, l1).
csa2_status check_layers(const csa2_layer_mode *modes, const csa2_layer_io *io, int32_t L,
                         int32_t l0, int32_t l1, const csa2_dims *d) {
  if (!io || !d) return CSA2_ERR_INVALID_ARG;
  csa2_status rc = check_modes(modes, L);
  if (rc != CSA2_OK) return rc;
  for (int32_t l = l0; l < l1; ++l) {
    const csa2_layer_io &x = io[l];
    const csa2_layer_io &kv = io[modes[l].kv_src];
    const csa2_layer_io &ix = io[modes[l].idx_src];
    if (modes[l].mode != CSA2_REUSE) {
      rc = check_topk_args(x.q_idx, x.w, kv.k_idx, d->B, d->T, d->H_I, d->d_I, d->N, d->n_prior,
                           d->ratio, d->topk, x.idx, nullptr);
      if (rc != CSA2_OK) return rc;
      if (kv.k_exps && !aligned(kv.k_exps, 16)) return CSA2_ERR_INVALID_ARG;
      if (kv.k_exps && !fp4_shape_ok(d->T, d->H_I, d->d_I, d->N, d->n_prior))
        return CSA2_ERR_UNSUPPORTED;
    }
    if (modes[l].mode == CSA2_FULL && x.app_pos) {
      if (!x.app_src || !x.app_key || x.k_exps || !aligned(x.app_src, 16) ||
          !aligned(x.app_key, 16) || !aligned(x.app_pos, 8) || d->d_I % 16 != 0)
        return CSA2_ERR_INVALID_ARG;
    }
    // a pool layer reads its Full source's pool; that Full layer writes it
    const bool keeps_pool = modes[l].mode == CSA2_FULL && x.pool;
    if (modes[l].mode == CSA2_REINDEX_POOL || keeps_pool) {
      if (!pool_dims_ok(d) || kv.k_exps || !scan_shape_supported(d->H_I, d->d_I))
        return CSA2_ERR_UNSUPPORTED;
      if (!kv.pool || !aligned(kv.pool, 4)) return CSA2_ERR_INVALID_ARG;
    }
    rc = check_attn_args(x.q, kv.codes, kv.scales, ix.idx, x.win_k, x.win_v, d->B, d->T, d->H,
                         d->D, d->N, d->topk, d->W, x.out, x.lse);
    if (rc != CSA2_OK) return rc;
  }
  return CSA2_OK;
}

csa2_status run_layer(const csa2_layer_mode *modes, const csa2_layer_io *io, int32_t l,
                      const csa2_dims *d, void *ws, size_t ws_bytes, cudaStream_t st) {
  const csa2_layer_io &x = io[l];
  const csa2_layer_io &kv = io[modes[l].kv_src];
  const csa2_layer_io &ix = io[modes[l].idx_src];
  if (modes[l].mode == CSA2_REINDEX_POOL) {
    // the top-k within the Full source's pool, then attention with it
    const int64_t P = int64_t(d->pool_block) * d->pool_blocks;
    csa2_status rc = run_pool_topk(x.q_idx, x.w, kv.k_idx, d->B, d->H_I, d->d_I, d->N, kv.pool,
                                   (int32_t)P, d->topk, x.idx, ws, ws_bytes, st);
    if (rc != CSA2_OK) return rc;
    return run_attn(x.q, kv.codes, kv.scales, x.idx, x.win_k, x.win_v, d->B, d->T, d->H, d->D,
                    d->N, d->topk, d->W, d->sm_scale, x.out, x.lse, st);
  }
  if (modes[l].mode != CSA2_REUSE) {
    // Full / Reindex: scan this layer's index query over the kv store's keys,
    // then select and attend in one per-row cluster kernel.
    if (modes[l].mode == CSA2_FULL && x.app_pos) {  // this step's entry append first
      const int64_t units = int64_t(d->B) * (d->D / 16 + d->d_I / 16);
      TraceScope ts("append_entry", st);
      append_entry_kernel<<<(unsigned)std::min<int64_t>(ceil_div(units, 128), 1024), 128, 0, st>>>(
          x.app_src, x.app_key, x.app_pos, d->B, d->D, d->d_I, d->N,
          const_cast<uint8_t *>(x.codes), const_cast<float *>(x.scales),
          const_cast<int8_t *>(x.k_idx));
      if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
    }
    AttnArgs att{x.q, kv.codes, kv.scales, x.win_k, x.win_v, d->H, d->D, d->W, d->sm_scale,
                 x.out, x.lse};
    if (modes[l].mode == CSA2_FULL && x.pool) {  // the layer also keeps its candidate pool
      const size_t off = pool_ext_offset(d);
      const PoolExt X0 = pool_ext_layout(nullptr, d->B, d->N, d->pool_block, d->pool_blocks);
      if (ws_bytes < off + X0.bytes) return CSA2_ERR_WORKSPACE;
      PoolReq pr{d->pool_block, d->pool_blocks, x.pool,
                 pool_ext_layout(static_cast<char *>(ws) + off, d->B, d->N, d->pool_block,
                                 d->pool_blocks)};
      return run_index_topk(x.q_idx, x.w, kv.k_idx, kv.k_exps, d->B, d->T, d->H_I, d->d_I, d->N,
                            d->n_prior, d->ratio, d->topk, x.idx, nullptr, &att, ws, off, st,
                            &pr);
    }
    return run_index_topk(x.q_idx, x.w, kv.k_idx, kv.k_exps, d->B, d->T, d->H_I, d->d_I, d->N,
                          d->n_prior, d->ratio, d->topk, x.idx, nullptr, &att, ws, ws_bytes, st);
  }
  // Reuse: attend with the source layer's selection.
  return run_attn(x.q, kv.codes, kv.scales, ix.idx, x.win_k, x.win_v, d->B, d->T, d->H, d->D,
                  d->N, d->topk, d->W, d->sm_scale, x.out, x.lse, st);
}

}  // namespace

extern "C" {

csa2_status csa2_layer_run(const csa2_layer_mode *modes, const csa2_layer_io *io, int32_t L,
                           int32_t layer, const csa2_dims *d, void *ws, size_t ws_bytes,
                           void *stream) {
  if (layer < 0 || layer >= L) return CSA2_ERR_INVALID_ARG;
  csa2_status rc = check_layers(modes, io, L, layer, layer + 1, d);
  if (rc != CSA2_OK) return rc;
  if (int64_t(d->B) * d->T == 0) return CSA2_OK;
  const size_t need = csa2_layer_group_workspace_size(d);
  if (need == 0) return CSA2_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < need || !aligned(ws, 16)) return CSA2_ERR_WORKSPACE;
  return run_layer(modes, io, layer, d, ws, ws_bytes, as_stream(stream));
}

csa2_status csa2_layer_group_run(const csa2_layer_mode *modes, const csa2_layer_io *io, int32_t L,
                                 const csa2_dims *d, void *ws, size_t ws_bytes, void *stream) {
  csa2_status rc = check_layers(modes, io, L, 0, L, d);
  if (rc != CSA2_OK) return rc;
  if (int64_t(d->B) * d->T == 0) return CSA2_OK;
  const size_t need = csa2_layer_group_workspace_size(d);
  if (need == 0) return CSA2_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < need || !aligned(ws, 16)) return CSA2_ERR_WORKSPACE;
  for (int32_t l = 0; l < L; ++l) {
    rc = run_layer(modes, io, l, d, ws, ws_bytes, as_stream(stream));
    if (rc != CSA2_OK) return rc;
  }
  return CSA2_OK;
}

csa2_status csa2_trace_enable(int32_t enable) {
  trace_clear();
  g_trace_on = enable != 0;
  return CSA2_OK;
}

int32_t csa2_trace_count(void) { return (int32_t)g_trace_n; }

csa2_status csa2_trace_get(int32_t i, const char **name, float *ms) {
  if (i < 0 || (size_t)i >= g_trace_n || !name || !ms) return CSA2_ERR_INVALID_ARG;
  const TraceRecord &r = g_trace[i];
  if (cudaEventSynchronize(r.stop) != cudaSuccess ||
      cudaEventElapsedTime(ms, r.start, r.stop) != cudaSuccess) {
    cudaGetLastError();  // a failed query must not be reported by the next launch
    return CSA2_ERR_CUDA;
  }
  *name = r.name;
  return CSA2_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Index + top-k for callers that cannot allocate device memory.
// ---------------------------------------------------------------------------
// Fixed scratch in the library's own device memory: every GPU that loads the
// library keeps these 16 MiB until the process exits.  All calls share it.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of the scratch on the current device, looked up once per
// device (the name itself is only a host-side stand-in).  The address is
// that of the device's primary context (the one the CUDA runtime uses).
// Host threads may race on the first lookup: each stores the same address.
void *noalloc_scratch(csa2_status *rc) {
  static std::atomic<void *> addr[256];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) {
    *rc = CSA2_ERR_CUDA;
    return nullptr;
  }
  void *a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    if (cudaGetSymbolAddress(&a, g_noalloc_scratch) != cudaSuccess || !a) {
      *rc = CSA2_ERR_CUDA;
      return nullptr;
    }
    addr[dev].store(a, std::memory_order_release);
  }
  return a;
}

}  // namespace

extern "C" {

csa2_status csa2_index_topk_noalloc(const int8_t *q_idx, const float *w, const int8_t *k_idx,
                                    int32_t B, int32_t T, int32_t H_I, int32_t d_I, int64_t N,
                                    int64_t n_prior, int32_t ratio, int32_t topk,
                                    int32_t *idx_out, float *score_out, void *stream) {
  csa2_status rc = check_topk_args(q_idx, w, k_idx, B, T, H_I, d_I, N, n_prior, ratio, topk,
                                   idx_out, score_out);
  if (rc != CSA2_OK || int64_t(B) * T == 0) return rc;
  if (csa2_index_topk_workspace_size(B, T, H_I, d_I, N, topk) > kNoAllocScratchBytes)
    return CSA2_ERR_UNSUPPORTED;
  void *ws = noalloc_scratch(&rc);
  if (!ws) return rc;
  return run_index_topk(q_idx, w, k_idx, nullptr, B, T, H_I, d_I, N, n_prior, ratio, topk,
                        idx_out, score_out, nullptr, ws, kNoAllocScratchBytes, as_stream(stream));
}

csa2_status csa2_set_decode_kernel(int32_t kernel) {
  if (kernel != CSA2_DECODE_SCAN_CLUSTER && kernel != CSA2_DECODE_FUSED)
    return CSA2_ERR_INVALID_ARG;
  g_decode_kernel.store(kernel, std::memory_order_relaxed);
  return CSA2_OK;
}

int32_t csa2_get_decode_kernel(void) { return fused_enabled() ? CSA2_DECODE_FUSED
                                                              : CSA2_DECODE_SCAN_CLUSTER; }

csa2_status csa2_wait_timeout_selftest(int64_t limit_cycles, void *stream) {
  if (limit_cycles < 1 || limit_cycles > (int64_t(1) << 32)) return CSA2_ERR_INVALID_ARG;
  fd::wait_timeout_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>((long long)limit_cycles);
  return after_launch();
}

csa2_status csa2_get_device_status(void *stream, int32_t *code_out) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return CSA2_ERR_CUDA;
  uint32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return CSA2_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess)
    return CSA2_ERR_CUDA;
  if (code_out) *code_out = (int32_t)v;
  return v ? CSA2_ERR_DEVICE_STATUS : CSA2_OK;
}

}  // extern "C"
