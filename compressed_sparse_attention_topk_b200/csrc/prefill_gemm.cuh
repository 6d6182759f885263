// Chunked-prefill indexer + top-k on the 5th-generation tensor cores.
//
// For a chunk of T queries the indexer dot products of every (query, entry)
// pair form a dense int8 contraction ("Why Is DeepSeek V4.1 Flash So
// Fast?", section 4: the indexer scores every compressed position;
// "DeepSeek-V4.1-Flash", "Reading input and writing output": a prefill
// processes all input tokens at once).  The selection must still be exactly
// the top-k of the fp32 scores defined per head (exact int32 dots, then
// w-weighted fp32 sum, each product and sum rounded on its own), so the
// tensor cores only decide which entries can be ignored:
//
//  1. prep: per query row the head-combined query Q = sum_h w_h q_h (real
//     valued) is written as two int8 levels, Q ~ (256 Q1 + Q2) / sigma, with
//     a rigorous bound E on |approximate score - exact fp32 score| for any
//     int8 key (the level residual times 128, plus the fp32 evaluation error
//     of the exact score).
//  2. sample: tcgen05 kind::i8 products of both levels against every s-th
//     key give approximate scores of a strided sample.
//  3. theta: per row the j-th largest sampled value, j * s = 2k, minus
//     margins of the bound, is the filter threshold tau.
//  4. filter: the same tcgen05 kernel over all visible keys writes one bit
//     per (row, entry): approximate score >= tau.  Every entry whose exact
//     score reaches (tau - 1) / sigma + E is among the bits set; entries
//     not set are strictly below that value.
//  5. select: per row, the set entries are rescored exactly; if at least k
//     of them lie above the bound (or every visible entry is set), the
//     row's exact top-k lies among them and is selected there (radix
//     select on the order-preserving score key, ties to the lower index,
//     output ascending).  Otherwise the row is listed for
//  6. fallback: exact multi-pass radix selection over all visible keys.
// The result is the exact top-k in every case; the fallback only costs time
// (it is taken when the sample misjudges a row's distribution, e.g. when
// many scores are equal).
#pragma once
#include <cuda.h>
#include <limits.h>

#include "common.cuh"

namespace csa2 {
namespace pf {

constexpr int kQ = 128;                         // query rows per CTA (MMA M = TMEM lanes)
constexpr int kN = 128;                         // keys per tile (MMA N)
constexpr int kEpiWarps = 16;                   // 4 per TMEM lane quarter
constexpr int kGemmThreads = 32 * (2 + kEpiWarps);
constexpr int kTmemCols = 512;                  // 2 buffers x (level 1 | level 2) x 128
constexpr int kGroupTiles = 8;                  // tiles of mask words staged per write
constexpr int kAxisUnit = kGroupTiles * kN;     // key-range granularity of a CTA
constexpr int kBRing = 65536;                   // bytes of the key-tile ring
constexpr int32_t kTauAll = -(1 << 30);         // passes every key (|approx| < 2^30)
constexpr int kSampleMax = 8192;                // samples per row at most
constexpr int kThetaThreads = 256;
constexpr int kSelThreads = 512;

template <int DI>
struct GemmShape {
  static_assert(DI == 32 || DI == 64 || DI == 128, "index dim");
  static constexpr int KSTEPS = DI / 32;        // 32-byte K steps of one MMA
  static constexpr int A_BYTES = kQ * DI;       // one level of the query tile
  static constexpr int B_BYTES = kN * DI;       // one key tile
  static constexpr int STAGES = kBRing / B_BYTES;
  // K-major operand rows of DI bytes = one swizzle row: 32/64/128-byte swizzle
  static constexpr uint64_t LAYOUT = DI == 128 ? 2 : (DI == 64 ? 4 : 6);
  static constexpr uint64_t SBO = 8 * DI;       // bytes between 8-row groups
};

template <int DI>
struct GemmSmem {
  alignas(1024) uint8_t a[2][kQ * DI];
  alignas(1024) uint8_t b[kBRing];
  union {
    uint32_t stage[kQ][32];           // filter: mask words of up to 8 tiles; word w of row r at (w + r) & 31
    int32_t sbuf[kEpiWarps][32][33];  // sample: one warp's 32 rows x 32 values, transposed on write
  };
  uint64_t a_full;
  uint64_t full[GemmShape<DI>::STAGES], empty[GemmShape<DI>::STAGES];
  uint64_t acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  volatile uint32_t abort_flag;
  int32_t tau[kQ];
  int32_t vis[kQ];
};

// Dynamic shared memory of the GEMM kernel: the structure, its 1 KiB
// alignment, and padding so that only one CTA fits per SM (each CTA takes
// all 512 tensor-memory columns).
template <int DI>
constexpr size_t gemm_smem_bytes() {
  return sizeof(GemmSmem<DI>) + 1024 < 120 * 1024 ? 120 * 1024 : sizeof(GemmSmem<DI>) + 1024;
}

struct GemmParams {
  int64_t N;           // entries per sequence
  int32_t T;           // queries per sequence
  int64_t n_prior;     // < 0: all N visible; else query t sees n < n_prior + (t+1)/ratio
  int32_t ratio;
  int32_t b;           // sequence of this pass
  int32_t t_begin;     // first query of this pass
  int32_t t_count;     // queries of this pass
  int64_t split_len;   // key-axis positions per CTA (multiple of kAxisUnit)
  int64_t axis_len;    // key-axis positions of the pass (sample mode: samples)
  const int32_t *tau;  // filter: [t_count] thresholds
  uint32_t *bits;      // filter: [t_count][bits_pitch] words, bit j of word w = entry 32w + j
  int64_t bits_pitch;
  int32_t level_scale; // 256: weight of the first query level (a runtime value, so the
                       // combine compiles to a multiply-add on the FMA pipe)
  int32_t sstride;     // sample: entries between samples
  int32_t *smp;        // sample: [t_count][smp_pitch] approximate scores, INT_MIN if invisible
  int64_t smp_pitch;
};

__host__ __device__ __forceinline__ int64_t visible_count(int64_t N, int64_t n_prior, int32_t ratio,
                                                          int64_t t) {
  if (n_prior < 0) return N;
  const int64_t v = n_prior + (t + 1) / ratio;
  return v < N ? v : N;
}

// ---------------------------------------------------------------------------
// tcgen05 / TMA primitives.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_3d(void *smem, const CUtensorMap *map, int x, int y, int z,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3, %4}], [%5];" ::"r"(smem_u32(smem)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor: K-major rows of DI bytes, swizzled over
// DI bytes, 8-row groups SBO bytes apart (leading offset unused: one swizzle
// row covers the whole K extent of an MMA), descriptor version 1.
template <int DI>
__device__ __forceinline__ uint64_t smem_desc(const void *smem) {
  using S = GemmShape<DI>;
  const uint64_t addr = smem_u32(smem);
  return ((addr >> 4) & 0x3FFFull) | (1ull << 16) | ((S::SBO >> 4) << 32) | (1ull << 46) |
         (S::LAYOUT << 61);
}

// Instruction descriptor: s32 accumulator, s8 x s8, A and B K-major,
// N = kN, M = kQ.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kN >> 3) << 17) |
                            ((uint32_t)(kQ >> 4) << 24);

__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void named_bar(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// 32 consecutive 32-bit TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// The same 32-bit value into 32 consecutive TMEM columns of this warp's lanes.
__device__ __forceinline__ void tmem_st32_fill(uint32_t taddr, uint32_t x) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, "
      "%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(
          taddr),
      "r"(x)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Bounded wait that also gives up once another role has aborted.
template <int DI>
__device__ __forceinline__ bool role_wait(GemmSmem<DI> &sm, uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;  // no clock read on the fast path
  const long long start = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (sm.abort_flag) return false;
    if (clock64() - start > (1ll << 32)) {
      raise_status(kStatusWaitTimeout);
      sm.abort_flag = 1u;
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// 1. prep: two-level int8 combined query + error bound.  One warp per row.
// ---------------------------------------------------------------------------
template <int DI, int HI>
__global__ void __launch_bounds__(256) pf_prep_kernel(const int8_t *__restrict__ q_idx,
                                                      const float *__restrict__ w, int32_t T,
                                                      int32_t b, int32_t t_begin, int32_t t_count,
                                                      int8_t *__restrict__ qa,
                                                      double *__restrict__ sigma_out,
                                                      double *__restrict__ err_out) {
  constexpr int EPL = DI / 32;  // elements per lane
  const int lane = threadIdx.x & 31;
  const int lt = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (lt >= t_count) return;
  const int64_t r = (int64_t)b * T + t_begin + lt;
  float wh[HI];
#pragma unroll
  for (int h = 0; h < HI; ++h) wh[h] = w[r * HI + h];
  double Q[EPL];
  double absq[HI];
#pragma unroll
  for (int e = 0; e < EPL; ++e) Q[e] = 0.0;
#pragma unroll
  for (int h = 0; h < HI; ++h) {
    absq[h] = 0.0;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int q = q_idx[(r * HI + h) * DI + lane + 32 * e];
      Q[e] += (double)wh[h] * (double)q;
      absq[h] += (double)(q < 0 ? -q : q);
    }
  }
  double mx = 0.0;
#pragma unroll
  for (int e = 0; e < EPL; ++e) mx = fmax(mx, fabs(Q[e]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const double sigma = mx > 0.0 ? 32512.0 / mx : 1.0;
  double resid = 0.0, qabs = 0.0;
  int8_t *row = qa + (int64_t)lt * 2 * DI;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const double x = Q[e] * sigma;
    double q1 = rint(x / 256.0);
    q1 = fmin(127.0, fmax(-127.0, q1));
    double q2 = rint(x - 256.0 * q1);
    q2 = fmin(127.0, fmax(-127.0, q2));
    row[lane + 32 * e] = (int8_t)q1;
    row[DI + lane + 32 * e] = (int8_t)q2;
    resid += fabs(Q[e] - (256.0 * q1 + q2) / sigma);
    qabs += fabs(Q[e]);
  }
  double wq = 0.0;  // sum_h |w_h| * sum_i |q_hi|, partial per lane
#pragma unroll
  for (int h = 0; h < HI; ++h) wq += fabs((double)wh[h]) * absq[h];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    resid += __shfl_xor_sync(0xffffffffu, resid, o);
    qabs += __shfl_xor_sync(0xffffffffu, qabs, o);
    wq += __shfl_xor_sync(0xffffffffu, wq, o);
  }
  if (lane == 0) {
    // |key| <= 128 per element.  e1: level residual (plus double rounding of
    // Q itself); e2: fp32 recursive-sum error of the exact score, gamma_HI <=
    // (HI + 1) 2^-24, plus an absolute allowance for underflow.
    const double e1 = 128.0 * resid * (1.0 + 0x1p-40) + 128.0 * qabs * 0x1p-48;
    const double e2 = (HI + 1) * 0x1p-24 * 128.0 * wq * (1.0 + 0x1p-40) + 1e-30;
    sigma_out[lt] = sigma;
    err_out[lt] = (e1 + e2) * (1.0 + 0x1p-30) + 1e-9;
  }
}

// ---------------------------------------------------------------------------
// 2./4. the tensor-core pass (sample or filter).
// grid (key-axis splits, 128-row blocks of the pass); kGemmThreads threads.
// warp 0: TMA producer; warp 1: TMEM owner + MMA issuer; warps 2..17:
// epilogue (warp w reads TMEM lanes 32*(w%4).., columns 32*((w-2)/4).. of a
// tile).
// ---------------------------------------------------------------------------
template <int DI, bool SAMPLE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    pf_gemm_kernel(const __grid_constant__ CUtensorMap amap,
                   const __grid_constant__ CUtensorMap bmap, const GemmParams p) {
  using S = GemmShape<DI>;
  extern __shared__ __align__(1024) unsigned char pf_smem_raw[];
  GemmSmem<DI> &sm = *reinterpret_cast<GemmSmem<DI> *>(
      (reinterpret_cast<uintptr_t>(pf_smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int lt0 = blockIdx.y * kQ;
  const int lt_last = min(lt0 + kQ, p.t_count) - 1;
  const int64_t v_last = visible_count(p.N, p.n_prior, p.ratio, (int64_t)p.t_begin + lt_last);
  int64_t axis_end = v_last;
  if (SAMPLE) axis_end = min64((v_last + p.sstride - 1) / p.sstride, p.axis_len);
  const int64_t k_lo = (int64_t)blockIdx.x * p.split_len;
  const int64_t k_hi = min64(axis_end, k_lo + p.split_len);
  const int ntiles = k_hi > k_lo ? (int)((k_hi - k_lo + kN - 1) / kN) : 0;

  if (tid == 0) {
    mbar_init(&sm.a_full, 1);
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.acc_full[a], 1);
      mbar_init(&sm.acc_empty[a], kEpiWarps / 2);
    }
    sm.abort_flag = 0u;
    fence_barrier_init();
  }
  for (int i = tid; i < kQ; i += kGemmThreads) {
    const int lt = lt0 + i;
    const bool ok = lt < p.t_count;
    sm.vis[i] = ok ? (int32_t)visible_count(p.N, p.n_prior, p.ratio, (int64_t)p.t_begin + lt) : 0;
    sm.tau[i] = (!SAMPLE && ok) ? p.tau[lt] : kTauAll;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && ntiles > 0) {
      mbar_arrive_expect_tx(&sm.a_full, 2 * S::A_BYTES);
      tma_load_3d(sm.a[0], &amap, 0, 0, lt0, &sm.a_full);
      tma_load_3d(sm.a[1], &amap, 0, 1, lt0, &sm.a_full);
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % S::STAGES;
        if (t >= S::STAGES && !role_wait(sm, &sm.empty[s], (uint32_t)((t / S::STAGES) - 1) & 1u))
          break;
        mbar_arrive_expect_tx(&sm.full[s], S::B_BYTES);
        tma_load_3d(sm.b + s * S::B_BYTES, &bmap, 0, (int)(k_lo + (int64_t)t * kN), p.b,
                    &sm.full[s]);
        issued = t + 1;
      }
      if (sm.abort_flag) {  // copies still in flight must land before the CTA exits
        mbar_wait_bounded(&sm.a_full, 0u);
        for (int t = issued > S::STAGES ? issued - S::STAGES : 0; t < issued; ++t)
          mbar_wait_bounded(&sm.full[t % S::STAGES], (uint32_t)(t / S::STAGES) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && ntiles > 0) {
      const bool ok = role_wait(sm, &sm.a_full, 0u);
      const uint64_t a0 = smem_desc<DI>(sm.a[0]), a1 = smem_desc<DI>(sm.a[1]);
      int issued = 0;
      for (int t = 0; ok && t < ntiles; ++t) {
        const int s = t % S::STAGES, acc = t & 1;
        // buffer free: completion (t >> 1) of its barrier (the first one is the
        // epilogue's bias initialisation)
        if (!role_wait(sm, &sm.acc_empty[acc], (uint32_t)(t >> 1) & 1u)) break;
        if (!role_wait(sm, &sm.full[s], (uint32_t)(t / S::STAGES) & 1u)) break;
        tc_fence_after();
        const uint64_t bd = smem_desc<DI>(sm.b + s * S::B_BYTES);
        const uint32_t d1 = tmem + (uint32_t)(acc * 2 * kN), d2 = d1 + kN;
#pragma unroll
        for (int k = 0; k < S::KSTEPS; ++k) {  // +32 bytes per K step = +2 in the address field
          umma_i8(d1, a0 + 2 * k, bd + 2 * k, k > 0 ? 1u : 0u);
          umma_i8(d2, a1 + 2 * k, bd + 2 * k, 1u);  // onto the row's bias
        }
        umma_commit(&sm.empty[s]);
        umma_commit(&sm.acc_full[acc]);
        issued = t + 1;
      }
      if (issued > 0) {  // every product done before the tensor memory is freed
        const int t = issued - 1;
        mbar_wait_bounded(&sm.acc_full[t & 1], (uint32_t)(t >> 1) & 1u);
      }
    }
  } else if (ntiles > 0) {
    // ---------------- epilogue ----------------
    // Two groups of 8 warps (2 per TMEM lane quarter) take alternate tiles,
    // so one group's TMEM loads overlap the other's arithmetic; group g owns
    // accumulator buffer g.  A warp covers 64 columns (two 32-column chunks)
    // of its group's tiles.  Every epilogue warp runs the same loop of
    // 8-tile groups and the same quarter barriers, aborted or not, so the
    // barriers always complete.
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int grp = (ew >> 2) & 1;
    const int half = ew >> 3;
    const int row = quarter * 32 + lane;
    const int32_t vis = sm.vis[row];
    const int32_t tau = sm.tau[row];
    const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(grp * 2 * kN);
    const int32_t mul = p.level_scale;
    // The level-2 accumulator of every tile starts at the row's bias, -tau
    // (0 when sampling), so 256 v1 + v2 already is the difference to tau.
    const uint32_t bias = SAMPLE ? 0u : (uint32_t)(-tau);
    auto release = [&]() {  // bias stores done -> buffer free for the next MMA
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[grp]);
    };
    tmem_st32_fill(tbase + (uint32_t)(kN + half * 64), bias);
    tmem_st32_fill(tbase + (uint32_t)(kN + half * 64 + 32), bias);
    release();
    const int ngroups = (ntiles + kGroupTiles - 1) / kGroupTiles;
    for (int G = 0; G < ngroups; ++G) {
      const int t_end = min(ntiles, (G + 1) * kGroupTiles);
      for (int t = G * kGroupTiles + grp; t < t_end; t += 2) {
        // warp-uniform decision: the TMEM loads below are .sync.aligned
        const bool ok =
            __all_sync(0xffffffffu, role_wait(sm, &sm.acc_full[grp], (uint32_t)(t >> 1) & 1u));
        if (ok) tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          const int chunk = half * 2 + cc;  // 32-column chunk of the tile
          uint32_t v1[32], v2[32];
          if (ok) {
            tmem_ld32(tbase + (uint32_t)(chunk * 32), v1);
            tmem_ld32(tbase + (uint32_t)(kN + chunk * 32), v2);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v1[j] = v2[j] = 0u;
          }
          const int64_t c0 = k_lo + (int64_t)t * kN + chunk * 32;  // first key-axis position
          if constexpr (SAMPLE) {
            // through shared memory so that each row's 32 values leave as one line
            int32_t(*buf)[33] = sm.sbuf[ew];
#pragma unroll
            for (int j = 0; j < 32; ++j) buf[lane][j] = (int32_t)v1[j] * mul + (int32_t)v2[j];
            __syncwarp();
            const int64_t i = c0 + lane;
            for (int rr = 0; rr < 32; ++rr) {
              const int ltr = lt0 + quarter * 32 + rr;
              if (ltr < p.t_count && i < k_hi)
                p.smp[(int64_t)ltr * p.smp_pitch + i] =
                    (i * p.sstride < sm.vis[quarter * 32 + rr]) ? buf[rr][lane] : INT_MIN;
            }
            __syncwarp();
          } else {
            // bit j = (256 v1_j + v2_j - tau >= 0): shift the sign bits in,
            // highest column first, then invert
            uint32_t m = 0u;
#pragma unroll
            for (int j = 31; j >= 0; --j) {
              const int32_t d = (int32_t)v1[j] * mul + (int32_t)v2[j];  // 256 v1 + v2 - tau
              m = __funnelshift_l((uint32_t)d, m, 1);
            }
            m = ~m;
            if (c0 + 32 > vis) m = (c0 >= vis) ? 0u : (m & ((1u << (uint32_t)(vis - c0)) - 1u));
            const int wl = (t % kGroupTiles) * 4 + chunk;
            sm.stage[row][(wl + row) & 31] = m;
          }
        }
        if (ok) {  // (a TMEM store between the two chunks' loads would stall the second)
          tmem_st32_fill(tbase + (uint32_t)(kN + half * 64), bias);
          tmem_st32_fill(tbase + (uint32_t)(kN + half * 64 + 32), bias);
          release();
        }
      }
      if constexpr (!SAMPLE) {
        // the quarter's 32 rows x (tiles of this group x 4) words, 16 bytes
        // per thread, whole lines per row
        named_bar(1 + quarter, 128);
        const int nw = (t_end - G * kGroupTiles) * 4;
        const int64_t wb = (k_lo + (int64_t)G * kGroupTiles * kN) / 32;
        const int u = (ew >> 2) * 32 + lane;
        const int rr = quarter * 32 + (u >> 2);
        const int part = (u & 3) * 8;
        const int ltr = lt0 + rr;
        if (ltr < p.t_count) {
          uint32_t *dst = p.bits + (int64_t)ltr * p.bits_pitch + wb;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int w0 = part + 4 * h;
            if (w0 < nw) {
              uint4 o;
              o.x = sm.stage[rr][(w0 + rr) & 31];
              o.y = sm.stage[rr][(w0 + 1 + rr) & 31];
              o.z = sm.stage[rr][(w0 + 2 + rr) & 31];
              o.w = sm.stage[rr][(w0 + 3 + rr) & 31];
              *reinterpret_cast<uint4 *>(dst + w0) = o;
            }
          }
        }
        named_bar(1 + quarter, 128);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// 3. theta: filter threshold per row from the sampled approximate scores
// (kernel below, after the selection helper it shares with step 5).
// ---------------------------------------------------------------------------
struct ThetaParams {
  int64_t N;
  int64_t n_prior;
  int32_t ratio;
  int32_t t_begin, t_count;
  int32_t sstride;
  int64_t nsamp;        // samples per row written by the sample pass
  const int32_t *smp;
  int64_t smp_pitch;
  int32_t target;       // expected candidates: 2k
  int32_t cap;          // selection capacity per row
  const double *sigma, *err;
  int32_t *tau;
};

// ---------------------------------------------------------------------------
// Exact score of one entry (the definition used everywhere in the library).
// q: the row's H_I x DI int8 query as int4 chunks; w: its head weights.
// ---------------------------------------------------------------------------
template <int DI, int HI>
__device__ __forceinline__ float exact_score(const int8_t *krow, const int4 *q, const float *w) {
  int dot[HI];
#pragma unroll
  for (int h = 0; h < HI; ++h) dot[h] = 0;
#pragma unroll
  for (int c = 0; c < DI / 16; ++c) {
    const int4 kv = __ldg(reinterpret_cast<const int4 *>(krow) + c);
#pragma unroll
    for (int h = 0; h < HI; ++h) {
      const int4 qv = q[h * (DI / 16) + c];
      dot[h] = __dp4a(kv.x, qv.x, dot[h]);
      dot[h] = __dp4a(kv.y, qv.y, dot[h]);
      dot[h] = __dp4a(kv.z, qv.z, dot[h]);
      dot[h] = __dp4a(kv.w, qv.w, dot[h]);
    }
  }
  float acc = 0.0f;
#pragma unroll
  for (int h = 0; h < HI; ++h) acc = __fadd_rn(acc, __fmul_rn(w[h], __int2float_rn(dot[h])));
  return __fadd_rn(acc, 0.0f);
}

struct SelParams {
  const int8_t *q_idx;
  const float *w;
  const int8_t *k_idx;
  int64_t N;
  int32_t T;
  int64_t n_prior;
  int32_t ratio;
  int32_t b, t_begin, t_count;
  int32_t topk;
  int32_t cap;
  const uint32_t *bits;
  int64_t bits_pitch;
  const int32_t *tau;
  const double *sigma, *err;
  int32_t *idx;        // [B, T, topk]
  int32_t *fail_rows;  // rows handed to the fallback
  int32_t *fail_count;
};

template <int DI, int HI>
struct SelSmem {
  int4 q[HI * DI / 16];
  float w[HI];
  uint32_t hist[kBins1];
  uint32_t scratch[40];
  uint32_t res[2];
  // followed by cidx[cap], ckey[cap]
};

template <int DI, int HI>
__host__ __device__ constexpr size_t sel_head_bytes() {
  return (sizeof(SelSmem<DI, HI>) + 15) / 16 * 16;
}

// Block-wide threshold of the top `need` of n keys: the key kstar of the
// need-th largest and how many entries equal to it are taken (the rest of
// the taken entries are strictly above it).  Contains __syncthreads().
template <int THREADS>
__device__ void select_threshold(const uint32_t *ckey, int n, uint32_t need, uint32_t *hist,
                                 uint32_t *scratch, uint32_t *res, uint32_t &kstar,
                                 uint32_t &ties) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0u, left = need;
  for (int level = 0; level < 3; ++level) {
    for (int i = tid; i < kBins1; i += THREADS) hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += THREADS) {
      const uint32_t k = ckey[i];
      if (level == 0)
        atomicAdd(&hist[key_d1(k)], 1u);
      else if (level == 1) {
        if (key_d1(k) == prefix) atomicAdd(&hist[key_d2(k)], 1u);
      } else if ((k >> 10) == prefix)
        atomicAdd(&hist[key_d3(k)], 1u);
    }
    __syncthreads();
    if (level < 2)
      radix_threshold<THREADS, kBins1>(hist, left, scratch, res);
    else
      radix_threshold<THREADS, kBins3>(hist, left, scratch, res);
    const uint32_t bin = res[0];
    left -= res[1];
    prefix = level == 0 ? bin : (level == 1 ? (prefix << 11) | bin : (prefix << 10) | bin);
    __syncthreads();
  }
  kstar = prefix;
  ties = left;
}

// ---------------------------------------------------------------------------
// 3. theta kernel: the j-th largest sampled value, less margins of the
// bound.  One CTA of kThetaThreads per row.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThetaThreads) pf_theta_kernel(const ThetaParams p) {
  __shared__ uint32_t skey[kSampleMax];
  __shared__ uint32_t hist[kBins1];
  __shared__ uint32_t scratch[40];
  __shared__ uint32_t res[2];
  const int tid = threadIdx.x;
  const int lt = blockIdx.x;
  const int64_t V = visible_count(p.N, p.n_prior, p.ratio, (int64_t)p.t_begin + lt);
  const int64_t S_t = min64((V + p.sstride - 1) / p.sstride, p.nsamp);
  const int64_t j = (p.target + p.sstride - 1) / p.sstride;
  if (V <= p.cap || j > S_t) {  // select over every visible entry
    if (tid == 0) p.tau[lt] = kTauAll;
    return;
  }
  // order-preserving unsigned keys of the sampled int32 values
  const int32_t *row = p.smp + (int64_t)lt * p.smp_pitch;
  for (int i = tid; i < S_t; i += kThetaThreads) skey[i] = (uint32_t)row[i] ^ 0x80000000u;
  __syncthreads();
  uint32_t kstar, ties;
  select_threshold<kThetaThreads>(skey, (int)S_t, (uint32_t)j, hist, scratch, res, kstar, ties);
  if (tid == 0) {
    const int64_t theta = (int64_t)(int32_t)(kstar ^ 0x80000000u);
    const double es = p.err[lt] * p.sigma[lt];
    const int64_t margin = 3 * (int64_t)ceil(es) + 4;
    int64_t t = theta - margin;
    if (t < kTauAll) t = kTauAll;
    p.tau[lt] = (int32_t)t;
  }
}

// ---------------------------------------------------------------------------
// 5. select: candidates of a row -> exact rescoring -> exact top-k, or hand
// the row to the fallback.  One CTA of kSelThreads per row.
// ---------------------------------------------------------------------------
template <int DI, int HI>
__global__ void __launch_bounds__(kSelThreads, 2) pf_select_kernel(const SelParams p) {
  extern __shared__ __align__(16) unsigned char sel_smem_raw[];
  SelSmem<DI, HI> &sm = *reinterpret_cast<SelSmem<DI, HI> *>(sel_smem_raw);
  uint32_t *cidx = reinterpret_cast<uint32_t *>(sel_smem_raw + sel_head_bytes<DI, HI>());
  uint32_t *ckey = cidx + p.cap;
  const int tid = threadIdx.x;
  const int lt = blockIdx.x;
  const int64_t t = (int64_t)p.t_begin + lt;
  const int64_t r = (int64_t)p.b * p.T + t;
  const int64_t V = visible_count(p.N, p.n_prior, p.ratio, t);
  int32_t *orow = p.idx + r * p.topk;
  if (V <= 0) {
    for (int i = tid; i < p.topk; i += kSelThreads) orow[i] = -1;
    return;
  }
  const int4 *qsrc = reinterpret_cast<const int4 *>(p.q_idx + r * HI * DI);
  for (int i = tid; i < HI * DI / 16; i += kSelThreads) sm.q[i] = qsrc[i];
  if (tid < HI) sm.w[tid] = p.w[r * HI + tid];

  // candidates in ascending entry order: thread u owns a contiguous,
  // 16-byte aligned range of mask words; the first kWordsCached of them stay
  // in registers between the count and the extraction
  constexpr int kWordsCached = 16;
  const uint32_t *brow = p.bits + (int64_t)lt * p.bits_pitch;
  const int64_t nw = (V + 31) / 32;
  const int64_t wpt = ((nw + kSelThreads - 1) / kSelThreads + 3) & ~int64_t(3);
  const int64_t w0 = min64(nw, (int64_t)tid * wpt), w1 = min64(nw, w0 + wpt);
  const uint32_t last_mask = (V & 31) ? (1u << (uint32_t)(V & 31)) - 1u : 0xffffffffu;
  auto word = [&](int64_t wi, uint32_t raw) -> uint32_t {
    if (wi >= w1) return 0u;
    return wi == nw - 1 ? (raw & last_mask) : raw;
  };
  uint32_t wv[kWordsCached];
#pragma unroll
  for (int c = 0; c < kWordsCached / 4; ++c) {
    const int64_t wi = w0 + 4 * c;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (wi < w1) x = __ldg(reinterpret_cast<const uint4 *>(brow + wi));
    wv[4 * c] = word(wi, x.x);
    wv[4 * c + 1] = word(wi + 1, x.y);
    wv[4 * c + 2] = word(wi + 2, x.z);
    wv[4 * c + 3] = word(wi + 3, x.w);
  }
  uint32_t cnt = 0;
#pragma unroll
  for (int c = 0; c < kWordsCached; ++c) cnt += __popc(wv[c]);
  for (int64_t wi = w0 + kWordsCached; wi < w1; wi += 4) {  // rows longer than 512 x 32 words
    const uint4 x = __ldg(reinterpret_cast<const uint4 *>(brow + wi));
    cnt += __popc(word(wi, x.x)) + __popc(word(wi + 1, x.y)) + __popc(word(wi + 2, x.z)) +
           __popc(word(wi + 3, x.w));
  }
  uint32_t C;
  uint32_t pos = block_excl_scan<kSelThreads>(cnt, sm.scratch, C);
  const bool overflow = C > (uint32_t)p.cap;
  if (!overflow) {
#pragma unroll
    for (int c = 0; c < kWordsCached; ++c) {
      uint32_t m = wv[c];
      while (m) {
        cidx[pos++] = (uint32_t)((w0 + c) * 32 + (__ffs(m) - 1));
        m &= m - 1u;
      }
    }
    for (int64_t wi = w0 + kWordsCached; wi < w1; wi += 4) {
      const uint4 x = __ldg(reinterpret_cast<const uint4 *>(brow + wi));
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
      for (int e = 0; e < 4; ++e) {
        uint32_t m = word(wi + e, xs[e]);
        while (m) {
          cidx[pos++] = (uint32_t)((wi + e) * 32 + (__ffs(m) - 1));
          m &= m - 1u;
        }
      }
    }
  }
  __syncthreads();
  bool fail = overflow;
  if (!fail) {
    // exact scores, two candidates per thread in flight; count those
    // certified above every entry left out
    const double U = ((double)p.tau[lt] - 1.0) / p.sigma[lt] + p.err[lt];
    const int8_t *kseq = p.k_idx + (int64_t)p.b * p.N * DI;
    uint32_t above = 0;
    for (uint32_t i0 = tid; i0 < C; i0 += 2 * kSelThreads) {
      float s[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t i = i0 + u * kSelThreads;
        s[u] = i < C ? exact_score<DI, HI>(kseq + (int64_t)cidx[i] * DI, sm.q, sm.w) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t i = i0 + u * kSelThreads;
        if (i < C) {
          ckey[i] = score_key(s[u]);
          above += (double)s[u] > U;
        }
      }
    }
    uint32_t total_above;
    block_excl_scan<kSelThreads>(above, sm.scratch, total_above);
    fail = (int64_t)C < V && total_above < (uint32_t)p.topk;
  }
  if (fail) {
    if (tid == 0) {
      const int slot = atomicAdd(p.fail_count, 1);
      p.fail_rows[slot] = lt;
    }
    return;
  }
  const uint32_t need = min((uint32_t)p.topk, C);
  uint32_t kstar = 0u, ties = C;  // all taken when C <= need: every key >= 0 ...
  bool all = C <= need;
  if (!all) select_threshold<kSelThreads>(ckey, (int)C, need, sm.hist, sm.scratch, sm.res, kstar, ties);
  // ordered write: thread u takes candidates [u*per, (u+1)*per)
  const int per = (int)((C + kSelThreads - 1) / kSelThreads);
  const int i0 = min((int)C, tid * per), i1 = min((int)C, i0 + per);
  uint32_t nt = 0;
  if (!all)
    for (int i = i0; i < i1; ++i) nt += ckey[i] == kstar;
  uint32_t tot;
  uint32_t tie_rank = block_excl_scan<kSelThreads>(nt, sm.scratch, tot);
  uint32_t ns = 0;
  {
    uint32_t tr = tie_rank;
    for (int i = i0; i < i1; ++i) {
      if (all) {
        ++ns;
        continue;
      }
      const uint32_t k = ckey[i];
      if (k > kstar)
        ++ns;
      else if (k == kstar) {
        if (tr < ties) ++ns;
        ++tr;
      }
    }
  }
  uint32_t opos = block_excl_scan<kSelThreads>(ns, sm.scratch, tot);
  for (int i = i0; i < i1; ++i) {
    bool take = true;
    if (!all) {
      const uint32_t k = ckey[i];
      take = k > kstar;
      if (k == kstar) {
        take = tie_rank < ties;
        ++tie_rank;
      }
    }
    if (take) orow[opos++] = (int32_t)cidx[i];
  }
  for (int i = (int)need + tid; i < p.topk; i += kSelThreads) orow[i] = -1;
}

// ---------------------------------------------------------------------------
// 6. fallback: exact top-k of listed rows straight from the keys (three
// histogram passes over all visible entries, then an ordered output pass).
// grid: a fixed number of CTAs striding over the list.
// ---------------------------------------------------------------------------
template <int DI, int HI>
__global__ void __launch_bounds__(kSelThreads) pf_fallback_kernel(const SelParams p) {
  __shared__ int4 q[HI * DI / 16];
  __shared__ float wsh[HI];
  __shared__ uint32_t hist[kBins1];
  __shared__ uint32_t scratch[40];
  __shared__ uint32_t res[2];
  __shared__ uint32_t carry[2];
  const int tid = threadIdx.x;
  const int nfail = *reinterpret_cast<volatile int32_t *>(p.fail_count);
  const int8_t *kseq = p.k_idx + (int64_t)p.b * p.N * DI;
  for (int f = blockIdx.x; f < nfail; f += gridDim.x) {
    const int lt = p.fail_rows[f];
    const int64_t t = (int64_t)p.t_begin + lt;
    const int64_t r = (int64_t)p.b * p.T + t;
    const int64_t V = visible_count(p.N, p.n_prior, p.ratio, t);
    int32_t *orow = p.idx + r * p.topk;
    __syncthreads();  // the previous row is done with the shared arrays
    const int4 *qsrc = reinterpret_cast<const int4 *>(p.q_idx + r * HI * DI);
    for (int i = tid; i < HI * DI / 16; i += kSelThreads) q[i] = qsrc[i];
    if (tid < HI) wsh[tid] = p.w[r * HI + tid];
    __syncthreads();
    if (V <= p.topk) {
      for (int64_t i = tid; i < p.topk; i += kSelThreads) orow[i] = i < V ? (int32_t)i : -1;
      continue;
    }
    uint32_t prefix = 0u, left = (uint32_t)p.topk;
    for (int level = 0; level < 3; ++level) {
      for (int i = tid; i < kBins1; i += kSelThreads) hist[i] = 0u;
      __syncthreads();
      for (int64_t n = tid; n < V; n += kSelThreads) {
        const uint32_t k = score_key(exact_score<DI, HI>(kseq + n * DI, q, wsh));
        if (level == 0)
          atomicAdd(&hist[key_d1(k)], 1u);
        else if (level == 1) {
          if (key_d1(k) == prefix) atomicAdd(&hist[key_d2(k)], 1u);
        } else if ((k >> 10) == prefix)
          atomicAdd(&hist[key_d3(k)], 1u);
      }
      __syncthreads();
      if (level < 2)
        radix_threshold<kSelThreads, kBins1>(hist, left, scratch, res);
      else
        radix_threshold<kSelThreads, kBins3>(hist, left, scratch, res);
      const uint32_t bin = res[0];
      left -= res[1];
      prefix = level == 0 ? bin : (level == 1 ? (prefix << 11) | bin : (prefix << 10) | bin);
      __syncthreads();
    }
    const uint32_t kstar = prefix, ties = left;
    // ordered output in chunks of kSelThreads * PER consecutive entries
    if (tid == 0) carry[0] = carry[1] = 0u;  // ties seen, entries written
    __syncthreads();
    constexpr int PER = 8;
    for (int64_t base = 0; base < V; base += (int64_t)kSelThreads * PER) {
      const int64_t n0 = base + (int64_t)tid * PER;
      uint32_t k[PER];
      uint32_t nt = 0;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int64_t n = n0 + e;
        k[e] = n < V ? score_key(exact_score<DI, HI>(kseq + n * DI, q, wsh)) : 0u;
        nt += (n < V) && k[e] == kstar;
      }
      const uint32_t c0 = carry[0], c1 = carry[1];
      uint32_t tot;
      uint32_t tr = c0 + block_excl_scan<kSelThreads>(nt, scratch, tot);
      uint32_t ns = 0;
      {
        uint32_t x = tr;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          if (n0 + e >= V) continue;
          if (k[e] > kstar)
            ++ns;
          else if (k[e] == kstar) {
            if (x < ties) ++ns;
            ++x;
          }
        }
      }
      uint32_t tot2;
      uint32_t pos = c1 + block_excl_scan<kSelThreads>(ns, scratch, tot2);
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        if (n0 + e >= V) continue;
        bool take = k[e] > kstar;
        if (k[e] == kstar) {
          take = tr < ties;
          ++tr;
        }
        if (take && pos < (uint32_t)p.topk) orow[pos++] = (int32_t)(n0 + e);
      }
      __syncthreads();
      if (tid == 0) {
        carry[0] = c0 + tot;
        carry[1] = c1 + tot2;
      }
      __syncthreads();
    }
  }
}

}  // namespace pf
}  // namespace csa2
