// C ABI of the CSA2 hot path (see include/csa2.h for the contract of every
// entry point).  One translation unit: every kernel of the library is
// included here so that they share the device status word.
#include "csa2.h"

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "attention.cuh"
#include "common.cuh"
#include "index_scan.cuh"
#include "pack.cuh"
#include "topk.cuh"

using namespace csa2;

namespace {

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static int cache[256] = {0};
  if (dev >= 0 && dev < 256 && cache[dev]) return cache[dev];
  int v = 148;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) v = 148;
  if (dev >= 0 && dev < 256) cache[dev] = v;
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
    cudaEventRecord(r.start, st);
  }
  ~TraceScope() {
    if (rec) cudaEventRecord(rec->stop, st);
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

int topk_regions(int64_t N) {
  return (int)std::min<int64_t>(kMaxRegions, std::max<int64_t>(1, ceil_div(N, kSelSpan)));
}

struct TopkWs {
  float *scores;
  uint2 *cand;
  uint32_t *hist1, *hist2, *cnt;
  size_t bytes;
};

TopkWs topk_ws_layout(void *base, int64_t R, int64_t N, int G2) {
  TopkWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  const size_t o_scores = take(size_t(R) * N * 4);
  const size_t o_cand = take(size_t(R) * N * 8);
  const size_t o_hist = take(size_t(R) * (kBins1 + kBins2) * 4);
  const size_t o_cnt = take(size_t(R) * G2 * 4);
  char *p = static_cast<char *>(base);
  w.scores = reinterpret_cast<float *>(p + o_scores);
  w.cand = reinterpret_cast<uint2 *>(p + o_cand);
  w.hist1 = reinterpret_cast<uint32_t *>(p + o_hist);
  w.hist2 = w.hist1 + size_t(R) * kBins1;
  w.cnt = reinterpret_cast<uint32_t *>(p + o_cnt);
  w.bytes = off;
  return w;
}

template <int DI, int HI>
void launch_scan(dim3 grid, cudaStream_t st, const int8_t *q_idx, const float *w,
                 const int8_t *k_idx, int32_t T, int64_t N, int64_t n_prior, int32_t ratio,
                 int64_t row0, float *scores, uint32_t *hist1, int write_masked) {
  index_scan_kernel<DI, HI><<<grid, kScanThreads, 0, st>>>(q_idx, w, k_idx, T, N, n_prior, ratio,
                                                            row0, scores, hist1, write_masked);
}

using ScanLaunch = void (*)(dim3, cudaStream_t, const int8_t *, const float *, const int8_t *,
                            int32_t, int64_t, int64_t, int32_t, int64_t, float *, uint32_t *, int);

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
  return topk_ws_layout(nullptr, R, N, topk_regions(N)).bytes;
}

csa2_status run_index_topk(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B,
                           int32_t T, int32_t H_I, int32_t d_I, int64_t N, int64_t n_prior,
                           int32_t ratio, int32_t topk, int32_t *idx_out, float *score_out,
                           void *ws, size_t ws_bytes, cudaStream_t st) {
  const int64_t rows = int64_t(B) * T;
  const int64_t R = topk_rows_per_pass(rows, N);
  const int G2 = topk_regions(N);
  const TopkWs L0 = topk_ws_layout(nullptr, R, N, G2);
  if (!ws || ws_bytes < L0.bytes || !aligned(ws, 16)) return CSA2_ERR_WORKSPACE;
  const TopkWs L = topk_ws_layout(ws, R, N, G2);
  const ScanLaunch scan = pick_scan(d_I, H_I);
  if (!scan) return CSA2_ERR_UNSUPPORTED;
  const int sms = device_sms();

  for (int64_t row0 = 0; row0 < rows; row0 += R) {
    const int64_t nr = std::min<int64_t>(R, rows - row0);
    // hist1 and hist2 of all R rows are one contiguous block
    if (cudaMemsetAsync(L.hist1, 0, size_t(R) * (kBins1 + kBins2) * 4, st) != cudaSuccess)
      return CSA2_ERR_CUDA;
    float *scores = score_out ? score_out + row0 * N : L.scores;
    // scan: ~3 CTAs per SM in total, at least 256 keys per CTA
    const int64_t g_want = ceil_div(3 * sms, nr);
    const int64_t g_max = std::max<int64_t>(1, ceil_div(N, 256));
    const int G = (int)std::max<int64_t>(1, std::min(g_want, g_max));
    {
      TraceScope ts("index_scan", st);
      scan(dim3(G, (unsigned)nr), st, q_idx, w, k_idx, T, N, n_prior, ratio, row0, scores,
           L.hist1, score_out != nullptr);
    }
    if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
    {
      TraceScope ts("topk_select", st);
      topk_select_kernel<<<dim3(G2, (unsigned)nr), kSelThreads, 0, st>>>(
          scores, N, T, n_prior, ratio, row0, topk, L.hist1, L.hist2, L.cand, L.cnt);
    }
    if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
    {
      TraceScope ts("topk_finalize", st);
      topk_finalize_kernel<<<(unsigned)nr, kFinThreads, 0, st>>>(N, T, n_prior, ratio, row0,
                                                                 topk, L.hist1, L.hist2, L.cand,
                                                                 L.cnt, G2, idx_out);
    }
    if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
  }
  return CSA2_OK;
}

// ---------------------------------------------------------------------------
// Attention: shapes, workspace, launches.
// ---------------------------------------------------------------------------
constexpr int64_t kAttnMaxRowsPerLaunch = 65535;

struct AttnPlan {
  int64_t rows_per_launch;
  int n_chunks, splits, chunks_per_split, hgroups;
  size_t part_bytes;
};

AttnPlan attn_plan(int32_t B, int32_t T, int32_t H, int32_t D, int32_t topk, int32_t W) {
  AttnPlan p{};
  const int64_t rows = int64_t(B) * T;
  p.rows_per_launch = std::max<int64_t>(1, std::min<int64_t>(rows, kAttnMaxRowsPerLaunch));
  p.n_chunks = (int)(ceil_div(topk, kAttnKeys) + ceil_div(W, kAttnKeys));
  p.hgroups = (int)ceil_div(H, kAttnHeads);
  const int64_t want = ceil_div(2 * int64_t(device_sms()), p.rows_per_launch * p.hgroups);
  p.splits = (int)std::max<int64_t>(1, std::min<int64_t>(want, std::max(1, p.n_chunks)));
  p.chunks_per_split = (int)ceil_div(p.n_chunks, p.splits);
  if (p.chunks_per_split > 0) p.splits = (int)ceil_div(p.n_chunks, p.chunks_per_split);
  if (p.splits < 1) p.splits = 1;
  p.part_bytes = align_up(size_t(p.rows_per_launch) * H * p.splits * (D + 2) * 4, 256);
  return p;
}

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

template <int D>
csa2_status launch_attn(const AttnPlan &p, int64_t row0, int64_t nr, const uint16_t *q,
                        const uint8_t *codes, const float *scales, const int32_t *idx,
                        const uint16_t *win_k, const uint16_t *win_v, int32_t T, int32_t H,
                        int64_t N, int32_t topk, int32_t W, float q_scale, float *part,
                        float *out, float *lse, cudaStream_t st) {
  const size_t smem = sizeof(AttnSmem<D>);
  static bool attr_set[256] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 256 || !attr_set[dev]) {
    if (cudaFuncSetAttribute(sparse_attn_partial_kernel<D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return CSA2_ERR_CUDA;
    if (dev >= 0 && dev < 256) attr_set[dev] = true;
  }
  // Offset the row-indexed inputs so the kernel's row 0 is global row row0.
  // The kernel derives (b, t) from its row, so launches start on a
  // sequence boundary.
  const int64_t b0 = row0 / T;
  const uint16_t *q0 = q + row0 * H * (int64_t)D;
  const int32_t *idx0 = idx ? idx + row0 * (int64_t)topk : nullptr;
  const uint8_t *codes0 = codes ? codes + b0 * N * (D / 2) : nullptr;
  const float *scales0 = scales ? scales + b0 * N * (D / 16) : nullptr;
  const int64_t win_rows = int64_t(W) - 1 + T;
  const uint16_t *wk0 = win_k ? win_k + b0 * win_rows * D : nullptr;
  const uint16_t *wv0 = win_v ? win_v + b0 * win_rows * D : nullptr;
  {
    TraceScope ts("attn_partial", st);
    sparse_attn_partial_kernel<D>
        <<<dim3(p.splits, (unsigned)nr, p.hgroups), kAttnThreads, smem, st>>>(
            q0, codes0, scales0, idx0, wk0, wv0, T, H, N, topk, W, q_scale, p.chunks_per_split,
            part);
  }
  if (after_launch() != CSA2_OK) return CSA2_ERR_CUDA;
  const int64_t warps = nr * H;
  {
    TraceScope ts("attn_combine", st);
    sparse_attn_combine_kernel<D><<<(unsigned)ceil_div(warps, 8), 256, 0, st>>>(
        part, p.splits, warps, out + row0 * H * (int64_t)D, lse ? lse + row0 * H : nullptr);
  }
  return after_launch();
}

csa2_status run_attn(const uint16_t *q, const uint8_t *codes, const float *scales,
                     const int32_t *idx, const uint16_t *win_k, const uint16_t *win_v, int32_t B,
                     int32_t T, int32_t H, int32_t D, int64_t N, int32_t topk, int32_t W,
                     float sm_scale, float *out, float *lse, void *ws, size_t ws_bytes,
                     cudaStream_t st) {
  const int64_t rows = int64_t(B) * T;
  // Launch chunks start on sequence boundaries.
  AttnPlan p = attn_plan(B, T, H, D, topk, W);
  int64_t seq_per_launch = std::max<int64_t>(1, p.rows_per_launch / std::max(T, 1));
  if (T > kAttnMaxRowsPerLaunch) return CSA2_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < p.part_bytes || !aligned(ws, 16)) return CSA2_ERR_WORKSPACE;
  float *part = static_cast<float *>(ws);
  const float q_scale = sm_scale * 1.4426950408889634f;
  for (int64_t s0 = 0; s0 < B; s0 += seq_per_launch) {
    const int64_t ns = std::min<int64_t>(seq_per_launch, B - s0);
    const int64_t row0 = s0 * T, nr = ns * T;
    csa2_status rc =
        (D == 128) ? launch_attn<128>(p, row0, nr, q, codes, scales, idx, win_k, win_v, T, H, N,
                                      topk, W, q_scale, part, out, lse, st)
                   : launch_attn<64>(p, row0, nr, q, codes, scales, idx, win_k, win_v, T, H, N,
                                     topk, W, q_scale, part, out, lse, st);
    if (rc != CSA2_OK) return rc;
  }
  (void)rows;
  return CSA2_OK;
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
  return topk_ws_bytes(B, T, N);
}

csa2_status csa2_index_topk(const int8_t *q_idx, const float *w, const int8_t *k_idx, int32_t B,
                            int32_t T, int32_t H_I, int32_t d_I, int64_t N, int64_t n_prior,
                            int32_t ratio, int32_t topk, int32_t *idx_out, float *score_out,
                            void *ws, size_t ws_bytes, void *stream) {
  csa2_status rc = check_topk_args(q_idx, w, k_idx, B, T, H_I, d_I, N, n_prior, ratio, topk,
                                   idx_out, score_out);
  if (rc != CSA2_OK || int64_t(B) * T == 0) return rc;
  return run_index_topk(q_idx, w, k_idx, B, T, H_I, d_I, N, n_prior, ratio, topk, idx_out,
                        score_out, ws, ws_bytes, as_stream(stream));
}

size_t csa2_sparse_attn_workspace_size(int32_t B, int32_t T, int32_t H, int32_t D, int32_t topk,
                                       int32_t W) {
  if (B < 0 || T < 0 || H < 1 || (D != 64 && D != 128) || topk < 0 || W < 0) return 0;
  return attn_plan(B, T, H, D, topk, W).part_bytes;
}

csa2_status csa2_sparse_attn_decode(const uint16_t *q, const uint8_t *codes, const float *scales,
                                    const int32_t *idx, const uint16_t *win_k,
                                    const uint16_t *win_v, int32_t B, int32_t H, int32_t D,
                                    int64_t N, int32_t topk, int32_t W, float sm_scale, float *out,
                                    float *lse, void *ws, size_t ws_bytes, void *stream) {
  csa2_status rc = check_attn_args(q, codes, scales, idx, win_k, win_v, B, 1, H, D, N, topk, W,
                                   out, lse);
  if (rc != CSA2_OK || B == 0) return rc;
  return run_attn(q, codes, scales, idx, win_k, win_v, B, 1, H, D, N, topk, W, sm_scale, out, lse,
                  ws, ws_bytes, as_stream(stream));
}

csa2_status csa2_sparse_attn_prefill(const uint16_t *q, const uint8_t *codes, const float *scales,
                                     const int32_t *idx, const uint16_t *win_k,
                                     const uint16_t *win_v, int32_t B, int32_t T, int32_t H,
                                     int32_t D, int64_t N, int32_t topk, int32_t W,
                                     float sm_scale, float *out, float *lse, void *ws,
                                     size_t ws_bytes, void *stream) {
  csa2_status rc = check_attn_args(q, codes, scales, idx, win_k, win_v, B, T, H, D, N, topk, W,
                                   out, lse);
  if (rc != CSA2_OK || int64_t(B) * T == 0) return rc;
  return run_attn(q, codes, scales, idx, win_k, win_v, B, T, H, D, N, topk, W, sm_scale, out, lse,
                  ws, ws_bytes, as_stream(stream));
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
  const size_t a = csa2_index_topk_workspace_size(d->B, d->T, d->H_I, d->d_I, d->N, d->topk);
  const size_t b = csa2_sparse_attn_workspace_size(d->B, d->T, d->H, d->D, d->topk, d->W);
  if (a == 0 || b == 0) return 0;
  return std::max(a, b);
}

csa2_status csa2_layer_group_run(const csa2_layer_mode *modes, const csa2_layer_io *io, int32_t L,
                                 const csa2_dims *d, void *ws, size_t ws_bytes, void *stream) {
  if (!io || !d) return CSA2_ERR_INVALID_ARG;
  csa2_status rc = check_modes(modes, L);
  if (rc != CSA2_OK) return rc;
  // Validate every layer's pointers before enqueueing anything.
  for (int32_t l = 0; l < L; ++l) {
    const csa2_layer_io &x = io[l];
    const csa2_layer_io &kv = io[modes[l].kv_src];
    const csa2_layer_io &ix = io[modes[l].idx_src];
    if (modes[l].mode != CSA2_REUSE) {
      rc = check_topk_args(x.q_idx, x.w, kv.k_idx, d->B, d->T, d->H_I, d->d_I, d->N, d->n_prior,
                           d->ratio, d->topk, x.idx, nullptr);
      if (rc != CSA2_OK) return rc;
    }
    rc = check_attn_args(x.q, kv.codes, kv.scales, ix.idx, x.win_k, x.win_v, d->B, d->T, d->H,
                         d->D, d->N, d->topk, d->W, x.out, x.lse);
    if (rc != CSA2_OK) return rc;
  }
  if (int64_t(d->B) * d->T == 0) return CSA2_OK;
  const size_t need = csa2_layer_group_workspace_size(d);
  if (need == 0) return CSA2_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < need || !aligned(ws, 16)) return CSA2_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  for (int32_t l = 0; l < L; ++l) {
    const csa2_layer_io &x = io[l];
    const csa2_layer_io &kv = io[modes[l].kv_src];
    const csa2_layer_io &ix = io[modes[l].idx_src];
    if (modes[l].mode != CSA2_REUSE) {
      rc = run_index_topk(x.q_idx, x.w, kv.k_idx, d->B, d->T, d->H_I, d->d_I, d->N, d->n_prior,
                          d->ratio, d->topk, x.idx, nullptr, ws, ws_bytes, st);
      if (rc != CSA2_OK) return rc;
    }
    rc = run_attn(x.q, kv.codes, kv.scales, ix.idx, x.win_k, x.win_v, d->B, d->T, d->H, d->D,
                  d->N, d->topk, d->W, d->sm_scale, x.out, x.lse, ws, ws_bytes, st);
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
  if (cudaEventSynchronize(r.stop) != cudaSuccess) return CSA2_ERR_CUDA;
  if (cudaEventElapsedTime(ms, r.start, r.stop) != cudaSuccess) return CSA2_ERR_CUDA;
  *name = r.name;
  return CSA2_OK;
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
