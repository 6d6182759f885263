// Common device helpers of the CSA2 kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace csa2 {

// ---------------------------------------------------------------------------
// Device status word: kernels never trap; they record what went wrong here
// and the host reads it back with csa2_get_device_status.
// ---------------------------------------------------------------------------
constexpr uint32_t kStatusBadIndex = 1u;     // an attention index >= N was skipped
constexpr uint32_t kStatusWaitTimeout = 2u;  // a bounded pipeline wait gave up

__device__ uint32_t g_device_status;

__device__ __forceinline__ void raise_status(uint32_t bit) { atomicOr(&g_device_status, bit); }

// ---------------------------------------------------------------------------
// Scores -> unsigned keys whose integer order is the float order.  The
// score producer never writes -0 or NaN, so equal scores give equal keys.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

__device__ __forceinline__ float bf16_to_f32_bits(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

// Radix digits of a key used by the top-k selection: 11 + 11 + 10 bits.
constexpr int kBins1 = 2048, kBins2 = 2048, kBins3 = 1024;
__device__ __forceinline__ uint32_t key_d1(uint32_t k) { return k >> 21; }
__device__ __forceinline__ uint32_t key_d2(uint32_t k) { return (k >> 10) & 2047u; }
__device__ __forceinline__ uint32_t key_d3(uint32_t k) { return k & 1023u; }

// ---------------------------------------------------------------------------
// Loads with explicit cache behaviour.
// ---------------------------------------------------------------------------
// Streamed once: keep out of L1, prefetch the 256-byte L2 line.
__device__ __forceinline__ int4 ld_stream_v4(const void *p) {
  int4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ---------------------------------------------------------------------------
// mbarrier + bulk-copy helpers with bounded waits.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking tests of a phase: a thread that polls with test_wait is never
// suspended, so it sees the phase complete as soon as it does (a try_wait
// that suspends the thread can resume it well after completion).  The
// cluster form acquires at cluster scope: data that other CTAs of the
// cluster delivered with st.async (below) is visible once the phase is seen
// complete.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_test_wait_cluster(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Shared-memory address of `p` (an address of this CTA's shared memory) in
// CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void *p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}

// Stores into the shared memory of CTA `rank` (at the offset of `dst` here)
// whose bytes are counted on the mbarrier at the offset of `bar` in that
// CTA (st.async with complete_tx): the receiver announces the bytes it
// expects and waits for its own barrier, no cluster-wide barrier involved.
__device__ __forceinline__ void st_async_v4(void *dst, uint4 v, uint64_t *bar, uint32_t rank) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
      ::"r"(cluster_addr(dst, rank)), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w),
        "r"(cluster_addr(bar, rank))
      : "memory");
}
__device__ __forceinline__ void st_async_v2(void *dst, uint32_t a, uint32_t b, uint64_t *bar,
                                            uint32_t rank) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];"
      ::"r"(cluster_addr(dst, rank)), "r"(a), "r"(b), "r"(cluster_addr(bar, rank))
      : "memory");
}

// Arrive on the mbarrier at the offset of `bar` in CTA `rank` of the
// cluster.  Relaxed: the arrival carries no data (the data these barriers
// count travels by bulk copies, counted in bytes), so no earlier write of
// the thread needs to be ordered before it (a release would wait for them).
__device__ __forceinline__ void mbar_remote_arrive(uint64_t *bar, uint32_t rank) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                   cluster_addr(bar, rank))
               : "memory");
}

// Bulk copy (copy engine) of `bytes` from this CTA's shared memory at `src`
// into CTA `rank`'s shared memory at the offset of `dst`, counted in bytes
// on the mbarrier at the offset of `bar` in that CTA.  Addresses 16-byte
// aligned, bytes a multiple of 16.  The copy reads `src` asynchronously:
// the sender keeps `src` unchanged, and stays resident, until it knows the
// bytes have landed.
__device__ __forceinline__ void bulk_s2s_cluster(void *dst, const void *src, uint32_t bytes,
                                                 uint64_t *bar, uint32_t rank) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, "
      "[%3];" ::"r"(cluster_addr(dst, rank)),
      "r"(smem_u32(src)), "r"(bytes), "r"(cluster_addr(bar, rank))
      : "memory");
}

// Order this thread's earlier shared-memory writes before later reads of
// them by bulk copies (the async proxy); every writing thread fences, then a
// block barrier, then the copy is issued.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}


// Wait for the given phase parity for at most ~2^32 cycles (about 2 s),
// polling without suspension; on timeout record it in the status word and
// return false.  The clock is read only once the phase is found incomplete:
// a clock read costs as much as ~150 cycles on the waiting thread's path.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  long long limit = (1ll << 32)) {
  if (mbar_test_wait(bar, parity)) return true;
  const long long start = clock64();
  while (!mbar_test_wait(bar, parity)) {
    if (clock64() - start > limit) {
      raise_status(kStatusWaitTimeout);
      return false;
    }
  }
  return true;
}

// Wait for a barrier that other CTAs of the cluster complete with st.async
// (below), with cluster-scope acquire: the bytes they stored into this CTA's
// shared memory are visible once the phase is seen complete.
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t *bar, uint32_t parity) {
  if (mbar_test_wait_cluster(bar, parity)) return true;
  const long long start = clock64();
  while (!mbar_test_wait_cluster(bar, parity)) {
    if (clock64() - start > (1ll << 32)) {
      raise_status(kStatusWaitTimeout);
      return false;
    }
  }
  return true;
}

// 1-D bulk copy global -> shared (TMA engine), completion counted in bytes
// on `bar`.  Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start before the previous kernel on its stream ends;
// it must wait before reading that kernel's results.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait_primary() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Warp / block reductions and scans.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ uint32_t lanemask_lt_u32() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Block-wide exclusive prefix sum of one value per thread; also returns the
// block total.  `scratch` holds >= 33 words.  Contains __syncthreads().
template <int THREADS>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *scratch,
                                                    uint32_t &total) {
  constexpr int NW = THREADS / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = warp_incl_scan(v);
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t s = (lane < NW) ? scratch[lane] : 0u;
    uint32_t si = warp_incl_scan(s);
    if (lane < NW) scratch[lane] = si - s;
    if (lane == NW - 1) scratch[32] = si;
  }
  __syncthreads();
  uint32_t excl = scratch[warp] + incl - v;
  total = scratch[32];
  __syncthreads();
  return excl;
}

// Radix threshold over a histogram of NBINS counts (in shared or global
// memory): the largest bin t with sum(hist[t..]) >= need, and the count of
// elements strictly above it.  When sum(hist) < need (only after an aborted
// producer) the result is bin 0 with the count above it, so that every CTA
// reading the same histogram still takes the same decisions.  Result in
// out[0] (bin) and out[1] (count above).  Contains __syncthreads().
template <int THREADS, int NBINS>
__device__ void radix_threshold(const uint32_t *hist, uint32_t need, uint32_t *scratch,
                                uint32_t *out) {
  static_assert(NBINS % THREADS == 0, "bins per thread");
  constexpr int BPT = NBINS / THREADS;
  const int tid = threadIdx.x;
  // Thread tid owns bins in descending order: rank tid covers bins
  // [NBINS - (tid+1)*BPT, NBINS - tid*BPT), so an ascending scan over threads
  // is a suffix scan over bins.
  const int hi = NBINS - tid * BPT;  // exclusive upper bin
  uint32_t local[BPT];
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < BPT; ++i) {
    local[i] = hist[hi - 1 - i];
    s += local[i];
  }
  if (tid == THREADS - 1) {  // default (sum < need): bin 0; bins [1, hi) of this thread counted below
    uint32_t a = 0;
    for (int i = 0; i < BPT - 1; ++i) a += local[i];
    out[0] = 0u;
    out[1] = a;  // completed by the scan below
  }
  uint32_t total;
  uint32_t above = block_excl_scan<THREADS>(s, scratch, total);
  if (tid == THREADS - 1 && total < need) out[1] += above;
  if (above < need && above + s >= need) {
    uint32_t acc = above;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      if (acc + local[i] >= need) {
        out[0] = static_cast<uint32_t>(hi - 1 - i);
        out[1] = acc;
        break;
      }
      acc += local[i];
    }
  }
  __syncthreads();
}

}  // namespace csa2
