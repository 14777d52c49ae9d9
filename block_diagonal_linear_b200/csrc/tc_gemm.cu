// Generic tcgen05 GEMM for the Monarch passes that are (batched, gathered) GEMMs:
//
//   D[m][n] = sum_k A[m][k] * B[n][k]     128 x BN tiles, bf16 operands, fp32 in TMEM.
//
// Two kinds of job share the kernel:
//   kind 0, block-diagonal stage (K-major operands): A is a row tile of an activation
//     matrix (rows x cols, K contiguous), B a weight block W[b] (N x K, the nn.Linear
//     layout); D is rounded to bf16 and written with TMA stores into a column range of
//     the output.  The A columns of one unit may be gathered from several 64-column
//     groups (col = b*a_b + (kb / a_grp)*a_gs + (kb % a_grp)*64), which lets a stage read
//     its input through a permutation whose groups are 64 columns wide without a pass
//     over memory.
//   kind 1, weight gradient (MN-major operands, rows of the activations are K): for a
//     group of blocks, A = act1[rows][cols] and B = act2[rows][cols], so
//     D[m][n] = sum_r act1[r][m] act2[r][n]; the rows are split into chunks (split-K) and
//     each unit writes the diagonal blocks of D (m and n in the same block) as fp32
//     partials, summed in a fixed order by a separate kernel.  One launch may carry two
//     such jobs (dR and dL of a backward): the units of the second follow those of the
//     first, with their own operand maps.
//   kind 2, block-diagonal stage, weight-stationary: as kind 0, but every CTA owns one
//     (batch b, n tile) pair and a contiguous range of m tiles; its weight tile W[b] (BN x K)
//     is loaded once and stays in shared memory, only A streams through the ring.  For
//     stages whose weight tile is reused by many row tiles (few blocks, many rows) this cuts
//     the L2 -> SM traffic per output tile roughly in half or better.
// Roles: warp 0 TMA producer, warp 1 MMA issuer and TMEM owner, warps 2..5 epilogue
// (one TMEM lane quadrant each: one D row per thread).  Operands move by TMA with 128B
// swizzle into a ring of stages; two TMEM accumulator slots let the epilogue of one unit
// overlap the MMAs of the next.  All waits are bounded (tc_common.cuh).
#include "tc_common.cuh"
#include "tc_gemm.cuh"

namespace monarch {

// CTA-pair kernels (tc_pair.cu).  launch_wgrad_pair: the caller builds 3-D operand maps whose B
// box is two 64-column chunks.  gemm_bd_pair: a kind-0 job with BN = 256 (maps built inside).
cudaError_t launch_wgrad_pair(const CUtensorMap& mA, const CUtensorMap& mB, GemmJob job, const CUtensorMap& mA2,
                              const CUtensorMap& mB2, GemmJob job2, float* partial, int* status, cudaStream_t st,
                              bool pdl);
cudaError_t gemm_bd_pair(const void* A, int64_t rows, int64_t a_cols, const void* W, int64_t w_rows, int K, void* Y,
                         int64_t y_cols, GemmJob job, int* status, cudaStream_t st, bool pdl);

constexpr int kGemmThreads = 192;
constexpr int kGemmEpiWarps = 4;

template <int BN_, int KIND_, int KBOX_ = 0>
struct GemmCfg {
  static constexpr int BN = BN_, KIND = KIND_, KBOX = KBOX_;
  static constexpr int BM = 128;
  static constexpr int A_BYTES = BM * 128;          // 128 x 64 bf16 (K-major) or 2 x (64 x 64) (MN-major)
  static constexpr int B_BYTES = KIND == 2 ? 0 : BN * 128;  // BN x 64 (K-major) or BN/64 x (64 x 64) (MN-major)
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STG_BYTES = KIND != 1 ? 2 * BM * 128 : 0;  // two 128 x 64 output chunks
  static constexpr int W_BYTES = KIND == 2 ? KBOX * BN * 128 : 0;  // kind 2: resident weight tile
  static constexpr int TMEM_COLS = 2 * BN <= 32 ? 32 : (2 * BN <= 64 ? 64 : (2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512)));
  static constexpr int NSTAGE_RAW = (kSmemBudget - STG_BYTES - W_BYTES - 1024) / STAGE;
  static constexpr int NSTAGE = NSTAGE_RAW > 8 ? 8 : NSTAGE_RAW;
  static constexpr int SMEM_BYTES = STG_BYTES + W_BYTES + NSTAGE * STAGE + 1024 + 1024;
  static_assert(BN % 64 == 0 && BN <= 256, "BN");
  static_assert(NSTAGE >= 2, "shared memory");
  static_assert(KIND != 2 || KBOX >= 1, "kind 2 needs the K extent");
};

struct GemmBars {
  uint64_t full[8], empty[8];
  uint64_t wfull;  // kind 2: the resident weight tile
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

// Unit index -> coordinates.  Kind 0: n tile fastest, then batch, then m tile (the units of
// one row tile run together, so its A tile is re-read from L2).  Kind 1: m, n tiles, then
// group, then split.
struct UnitCoord {
  int b, mt, nt, split;
  int second;  // kind 1: the unit belongs to the launch's second job
};
__device__ __forceinline__ UnitCoord unit_coord(const GemmJob& j, int64_t u) {
  UnitCoord c;
  c.nt = (int)(u % j.ntiles);
  u /= j.ntiles;
  if (j.kind == 0) {
    c.b = (int)(u % j.nb);
    c.mt = (int)(u / j.nb);
    c.split = 0;
  } else {
    c.mt = (int)(u % j.mtiles);
    u /= j.mtiles;
    c.b = (int)(u % j.nb);
    c.split = (int)(u / j.nb);
  }
  c.second = 0;
  return c;
}

// Units of this CTA: i = 0, 1, ... < unit_count().  Kinds 0 and 1: unit blockIdx.x + i*gridDim.x
// of the job (kind 1: of the two jobs' units, the second job's after the first's).  Kind 2: the CTA's (b, n tile) pair is blockIdx.x % (nb*ntiles) and its m tiles a
// contiguous range (the grid is a multiple of nb*ntiles).
__device__ __forceinline__ void kind2_range(const GemmJob& j, int* b, int* nt, int* lo, int* hi) {
  const int nwg = j.nb * j.ntiles;
  const int wg = (int)(blockIdx.x % nwg), ci = (int)(blockIdx.x / nwg), cpw = (int)(gridDim.x / nwg);
  *b = wg / j.ntiles;
  *nt = wg % j.ntiles;
  *lo = (int)((int64_t)ci * j.mtiles / cpw);
  *hi = (int)((int64_t)(ci + 1) * j.mtiles / cpw);
}
__device__ __forceinline__ int64_t unit_count(const GemmJob& j, const GemmJob& j2) {
  if (j.kind == 2) {
    int b, nt, lo, hi;
    kind2_range(j, &b, &nt, &lo, &hi);
    return hi - lo;
  }
  const int64_t total = j.units + (j.kind == 1 ? j2.units : 0);
  return total > (int64_t)blockIdx.x ? (total - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
}
__device__ __forceinline__ UnitCoord unit_at(const GemmJob& j, const GemmJob& j2, int64_t i) {
  if (j.kind == 2) {
    int b, nt, lo, hi;
    kind2_range(j, &b, &nt, &lo, &hi);
    UnitCoord c;
    c.b = b;
    c.nt = nt;
    c.mt = lo + (int)i;
    c.split = 0;
    c.second = 0;
    return c;
  }
  const int64_t g = blockIdx.x + i * gridDim.x;
  if (j.kind == 1 && g >= j.units) {
    UnitCoord c = unit_coord(j2, g - j.units);
    c.second = 1;
    return c;
  }
  return unit_coord(j, g);
}

// Number of 64-wide K stages of a unit.
__device__ __forceinline__ int unit_kstages(const GemmJob& j, const UnitCoord& c) {
  if (j.kind != 1) return j.kboxes;
  const int64_t r0 = (int64_t)c.split * j.split_rows;
  int64_t n = j.rows - r0;
  if (n > j.split_rows) n = j.split_rows;
  return (int)((n + 63) / 64);
}

template <class C>
__global__ void __launch_bounds__(kGemmThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmY, const __grid_constant__ GemmJob job,
                   const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                   const __grid_constant__ GemmJob job2, float* __restrict__ partial, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stg = smem;                      // kinds 0, 2: two 16 KB output staging chunks
  uint8_t* wreg = smem + C::STG_BYTES;      // kind 2: resident weight tile (KBOX boxes of BN x 64)
  uint8_t* ring = wreg + C::W_BYTES;
  GemmBars* bars = (GemmBars*)(ring + C::NSTAGE * C::STAGE);
  int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t nmine = unit_count(job, job2);  // units of this CTA

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      ptx::mbar_init(&bars->full[i], 1);
      ptx::mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->acc_full[i], 1);
      ptx::mbar_init(&bars->acc_empty[i], kGemmEpiWarps);
    }
    ptx::mbar_init(&bars->mma_done, 1);
    ptx::mbar_init(&bars->wfull, 1);
    bars->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // inputs may be written by the previous kernel of the stream
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      ptx::tma_prefetch_desc(&tmA);
      ptx::tma_prefetch_desc(&tmB);
      if (C::KIND != 1) ptx::tma_prefetch_desc(&tmY);
      if (C::KIND == 1 && job2.units > 0) {
        ptx::tma_prefetch_desc(&tmA2);
        ptx::tma_prefetch_desc(&tmB2);
      }
      const uint64_t pol = ptx::policy_evict_normal();
      if (C::KIND == 2 && nmine > 0) {
        const UnitCoord c0 = unit_at(job, job2, 0);
        ptx::mbar_arrive_expect_tx(&bars->wfull, C::W_BYTES);
        for (int kb = 0; kb < C::KBOX; ++kb)
          ptx::tma_load_2d(wreg + kb * (C::BN * 128), &tmB, &bars->wfull, kb * 64, c0.b * job.b_b + c0.nt * C::BN,
                           pol);
      }
      uint32_t it = 0;
      bool ok = true;
      for (int64_t i = 0; i < nmine && ok; ++i) {
        const UnitCoord c = unit_at(job, job2, i);
        const GemmJob& jb = c.second ? job2 : job;
        const CUtensorMap* mapA = c.second ? &tmA2 : &tmA;
        const CUtensorMap* mapB = c.second ? &tmB2 : &tmB;
        const int nk = unit_kstages(jb, c);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int st = it % C::NSTAGE;
          if (!wait_or_abort(&bars->empty[st], ((it / C::NSTAGE) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
          uint8_t* sa = ring + st * C::STAGE;
          uint8_t* sb = sa + C::A_BYTES;
          ptx::mbar_arrive_expect_tx(&bars->full[st], C::STAGE);
          if (C::KIND != 1) {
            const int ax = gcol(c.b, job.a_b, kb, job.a_grp, job.a_gs);
            ptx::tma_load_2d(sa, &tmA, &bars->full[st], ax, c.mt * C::BM, pol);
            if (C::KIND == 0) ptx::tma_load_2d(sb, &tmB, &bars->full[st], kb * 64, c.b * job.b_b + c.nt * C::BN, pol);
          } else {
            const int row = (int)((int64_t)c.split * jb.split_rows + (int64_t)kb * 64);
            const int ax = c.b * jb.a_b + c.mt * C::BM;
            if (jb.ab3d) {
              // one op per operand: TMA throughput per SM grows with the bytes per op (8 KB boxes
              // cap it near 50 GB/s, 16-32 KB ones reach 90-115 GB/s from L2)
              ptx::tma_load_3d(sa, mapA, &bars->full[st], 0, row, ax / 64, pol);
              ptx::tma_load_3d(sb, mapB, &bars->full[st], 0, row,
                               gcol(c.b, jb.b_b, c.nt * (C::BN / 64), jb.b_grp, jb.b_gs) / 64, pol);
            } else {
              ptx::tma_load_2d(sa, mapA, &bars->full[st], ax, row, pol);
              ptx::tma_load_2d(sa + 8192, mapA, &bars->full[st], ax + 64, row, pol);
#pragma unroll
              for (int h = 0; h < C::BN / 64; ++h)
                ptx::tma_load_2d(sb + h * 8192, mapB, &bars->full[st],
                                 gcol(c.b, jb.b_b, c.nt * (C::BN / 64) + h, jb.b_grp, jb.b_gs), row, pol);
            }
          }
        }
      }
      const uint32_t issued = it;
      for (uint32_t k = (issued > (uint32_t)C::NSTAGE ? issued - C::NSTAGE : 0); k < issued; ++k)
        ptx::mbar_wait_bounded(&bars->full[k % C::NSTAGE], (k / C::NSTAGE) & 1, kWaitLimitNs);
      if (C::KIND == 2 && nmine > 0) ptx::mbar_wait_bounded(&bars->wfull, 0, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    constexpr bool MN = C::KIND == 1;
    constexpr uint32_t idesc = make_idesc(C::BM, C::BN) | (MN ? (1u << 15) | (1u << 16) : 0u);
    // K-major: one 128-byte swizzled row per M/N index, a K step of 16 advances 32 bytes.
    // MN-major: one 128-byte row per K index holding 64 M/N indices (LBO = 8 KB between
    // the 64-wide M/N halves), a K step of 16 advances two 8-row groups (2 KB).
    const uint64_t dA = MN ? make_sdesc_lbo(ptx::smem_u32(ring), 8192, 1024, 2) : make_sdesc(ptx::smem_u32(ring), 1024, 2);
    const uint64_t dB = MN ? make_sdesc_lbo(ptx::smem_u32(ring + C::A_BYTES), 8192, 1024, 2)
                           : make_sdesc(ptx::smem_u32(C::KIND == 2 ? wreg : ring + C::A_BYTES), 1024, 2);
    constexpr uint64_t kstep = MN ? (2048 >> 4) : (32 >> 4);
    uint32_t it = 0, n = 0;
    bool ok = true;
    if (C::KIND == 2 && nmine > 0) ok = warp_wait_or_abort(lane, &bars->wfull, 0, abort_flag, status);
    for (int64_t i = 0; i < nmine && ok; ++i, ++n) {
      const UnitCoord c = unit_at(job, job2, i);
      const int nk = unit_kstages(c.second ? job2 : job, c);
      const int slot = n & 1;
      if (!warp_wait_or_abort(lane, &bars->acc_empty[slot], ((n >> 1) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
      ptx::tc_fence_after();
      const uint32_t d = tmem + slot * C::BN;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int st = it % C::NSTAGE;
        if (!warp_wait_or_abort(lane, &bars->full[st], (it / C::NSTAGE) & 1, abort_flag, status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint64_t soff = (uint64_t)((st * C::STAGE) >> 4);
        // kind 2: B is box kb of the resident weight tile
        const uint64_t boff = C::KIND == 2 ? (uint64_t)((kb * C::BN * 128) >> 4) : soff;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::mma_bf16_ss_elect(d, dA + soff + kk * kstep, dB + boff + kk * kstep, idesc,
                                 (kb > 0 || kk > 0) ? 1u : 0u);
        ptx::mma_commit_elect(&bars->empty[st]);
      }
      if (!ok) break;
      ptx::mma_commit_elect(&bars->acc_full[slot]);
    }
    ptx::mma_commit_elect(&bars->mma_done);
    if (lane == 0) wait_mma_done(&bars->mma_done, abort_flag, status);
    __syncwarp();
  } else {
    // ================================================================ epilogue (4 warps)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // D row of this thread
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool leader = (warp == 2 && lane == 0);
    const uint32_t stg_s = ptx::smem_u32(stg);
    uint32_t n = 0, chunk_n = 0;
    bool ok = true;
    for (int64_t i = 0; i < nmine && ok; ++i, ++n) {
      const UnitCoord c = unit_at(job, job2, i);
      const GemmJob& jb = c.second ? job2 : job;
      const int slot = n & 1;
      if (!wait_or_abort(&bars->acc_full[slot], (n >> 1) & 1, abort_flag, status)) { ok = false; break; }
      ptx::tc_fence_after();
      const uint32_t tb = tmem + lane_off + slot * C::BN;
      if (C::KIND != 1) {
        for (int ch = 0; ch < C::BN / 64; ++ch, ++chunk_n) {
          uint32_t v[64];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t t16[16];
            ptx::tmem_ld16(tb + ch * 64 + q * 16, t16);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[q * 16 + e] = t16[e];
          }
          ptx::tmem_wait_ld();
          const int sbuf = chunk_n & 1;
          // the TMA store that last read this staging buffer must have finished reading it
          if (leader) ptx::bulk_wait_read_allbut1();
          ptx::named_bar_sync(1, kGemmEpiWarps * 32);
          const uint32_t base = stg_s + sbuf * (C::BM * 128) + r * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            ptx::st_shared_v4(base + (((uint32_t)q ^ (uint32_t)(r & 7)) << 4),
                              ptx::pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1])),
                              ptx::pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                              ptx::pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                              ptx::pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
          ptx::fence_proxy_async_smem();
          ptx::named_bar_sync(1, kGemmEpiWarps * 32);
          if (leader) {
            ptx::tma_store_2d(&tmY, stg + sbuf * (C::BM * 128),
                              gcol(c.b, job.y_b, c.nt * (C::BN / 64) + ch, job.y_grp, job.y_gs), c.mt * C::BM);
            ptx::bulk_commit_group();
          }
        }
      } else {
        // diagonal blocks of D as fp32 partials: row m belongs to block blk = m_g / blk_a, and
        // its values go to the columns of that block, in logical column order (any column
        // permutation is applied when the partials are summed).  32-bit index math, one
        // division per unit, float4 stores.
        const int bla = (int)jb.blk_a, blb = (int)jb.blk_b;
        const int ma = c.b * jb.a_b + c.mt * C::BM + r;
        const int nb0 = c.b * jb.b_lb + c.nt * C::BN;
        const int blk = ma / bla;
        const bool row_ok = ma < (int)jb.a_cols;
        const int t_lo = max(0, blk * blb - nb0);
        const int t_hi = min(C::BN, min((blk + 1) * blb, (int)jb.b_cols) - nb0);
        // the warp's column range: from its first row's block to its last row's block
        const int ma0 = c.b * jb.a_b + c.mt * C::BM + quad * 32;
        const int w_lo = max(0, (ma0 / bla) * blb - nb0) & ~15;
        const int w_hi = min(C::BN, ((ma0 + 31) / bla + 1) * blb - nb0);
        float* prow = partial + (int64_t)c.split * jb.p_stride + jb.p_off + (int64_t)blk * bla * blb +
                      (int64_t)(ma - blk * bla) * blb + (nb0 - blk * blb);  // + tile column
        for (int c0 = w_lo; c0 < w_hi; c0 += 16) {
          uint32_t t16[16];
          ptx::tmem_ld16(tb + c0, t16);
          ptx::tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              const int cc = c0 + e;
              if (cc >= t_lo && cc < t_hi)
                *(float4*)(prow + cc) = make_float4(__uint_as_float(t16[e]), __uint_as_float(t16[e + 1]),
                                                    __uint_as_float(t16[e + 2]), __uint_as_float(t16[e + 3]));
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->acc_empty[slot]);
    }
    if (C::KIND != 1 && leader) ptx::bulk_wait_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int BN, int KIND, int KBOX = 0>
static cudaError_t launch_gemm_cfg(const CUtensorMap& mA, const CUtensorMap& mB, const CUtensorMap& mY,
                                   const GemmJob& job, const CUtensorMap& mA2, const CUtensorMap& mB2,
                                   const GemmJob& job2, float* partial, int* status, cudaStream_t st, bool pdl) {
  using C = GemmCfg<BN, KIND, KBOX>;
  cudaError_t e = ensure_smem_attr((const void*)tc_gemm_kernel<C>, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  int64_t grid;
  if (KIND == 2) {
    // CTAs per (b, n tile) pair: fill the SMs, at most one per m tile
    const int64_t nwg = (int64_t)job.nb * job.ntiles;
    int64_t cpw = num_sms() / nwg;
    if (cpw < 1) cpw = 1;
    if (cpw > job.mtiles) cpw = job.mtiles;
    grid = nwg * cpw;
  } else {
    const int64_t units = job.units + (KIND == 1 ? job2.units : 0);
    grid = num_sms();
    if (grid > units) grid = units;
  }
  return launch_kernel(tc_gemm_kernel<C>, dim3((unsigned)grid), dim3(kGemmThreads), C::SMEM_BYTES, st, pdl,
                       mA, mB, mY, job, mA2, mB2, job2, partial, status);
}

// One-job launch of the block-diagonal stage kinds (the second job is empty).
template <int BN, int KIND, int KBOX = 0>
static cudaError_t launch_stage_cfg(const CUtensorMap& mA, const CUtensorMap& mB, const CUtensorMap& mY,
                                    const GemmJob& job, int* status, cudaStream_t st, bool pdl) {
  const GemmJob none = {};
  return launch_gemm_cfg<BN, KIND, KBOX>(mA, mB, mY, job, mA, mB, none, nullptr, status, st, pdl);
}

cudaError_t gemm_bd(const void* A, int64_t rows, int64_t a_cols, const void* W, int64_t w_rows, int K,
                    void* Y, int64_t y_cols, int BN, GemmJob job, int* status, cudaStream_t st, bool pdl) {
  if (rows == 0) return cudaSuccess;
  // few rows (e.g. 1000): narrower N tiles, so that the units cover more of the SMs
  while (BN > 64 && (rows + 127) / 128 * job.nb * job.ntiles < num_sms() / 2) {
    BN /= 2;
    job.ntiles *= 2;
  }
  {
    // streamed 256-wide weight tiles (no resident configuration) with enough 256-row units to
    // fill the SM pairs: run on CTA pairs, each SM loading half of every weight stage
    const int64_t mt128 = (rows + 127) / 128, nwg = (int64_t)job.nb * job.ntiles;
    const bool stationary = mt128 >= 2 * ((num_sms() / nwg) > 0 ? (num_sms() / nwg) : 1);
    const bool resident = stationary && BN == 256 && (job.kboxes == 4 || job.kboxes == 2);
    if (BN == 256 && !resident && (rows + 255) / 256 * nwg >= num_sms() / 2)
      return gemm_bd_pair(A, rows, a_cols, W, w_rows, K, Y, y_cols, job, status, st, pdl);
  }
  CUtensorMap mA, mB, mY;
  if (!make_map_2d(&mA, A, (uint64_t)a_cols, (uint64_t)rows, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mB, W, (uint64_t)K, (uint64_t)w_rows, 64, (uint32_t)BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mY, Y, (uint64_t)y_cols, (uint64_t)rows, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  job.mtiles = (int)((rows + 127) / 128);
  job.units = (int64_t)job.mtiles * job.nb * job.ntiles;
  // weight-stationary when the (BN x K) weight tile fits the resident region and is reused by
  // at least two row tiles per CTA
  const int kbox = job.kboxes;
  const int64_t nwg = (int64_t)job.nb * job.ntiles;
  const bool stationary = (int64_t)job.mtiles >= 2 * ((num_sms() / nwg) > 0 ? (num_sms() / nwg) : 1);
  job.kind = 0;
  if (stationary) {
    job.kind = 2;
    if (BN == 256 && kbox == 4) return launch_stage_cfg<256, 2, 4>(mA, mB, mY, job, status, st, pdl);
    if (BN == 256 && kbox == 2) return launch_stage_cfg<256, 2, 2>(mA, mB, mY, job, status, st, pdl);
    if (BN == 128 && kbox == 8) return launch_stage_cfg<128, 2, 8>(mA, mB, mY, job, status, st, pdl);
    if (BN == 128 && kbox == 4) return launch_stage_cfg<128, 2, 4>(mA, mB, mY, job, status, st, pdl);
    if (BN == 128 && kbox == 2) return launch_stage_cfg<128, 2, 2>(mA, mB, mY, job, status, st, pdl);
    if (BN == 64 && kbox == 16) return launch_stage_cfg<64, 2, 16>(mA, mB, mY, job, status, st, pdl);
    if (BN == 64 && kbox == 4) return launch_stage_cfg<64, 2, 4>(mA, mB, mY, job, status, st, pdl);
    if (BN == 64 && kbox == 3) return launch_stage_cfg<64, 2, 3>(mA, mB, mY, job, status, st, pdl);
    if (BN == 64 && kbox == 2) return launch_stage_cfg<64, 2, 2>(mA, mB, mY, job, status, st, pdl);
    if (BN == 64 && kbox == 1) return launch_stage_cfg<64, 2, 1>(mA, mB, mY, job, status, st, pdl);
    job.kind = 0;  // no resident configuration for this tile: stream the weights
  }
  switch (BN) {
    case 64: return launch_stage_cfg<64, 0>(mA, mB, mY, job, status, st, pdl);
    case 128: return launch_stage_cfg<128, 0>(mA, mB, mY, job, status, st, pdl);
    case 256: return launch_stage_cfg<256, 0>(mA, mB, mY, job, status, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

// Operand maps of one weight-gradient job; sets job.ab3d, kind, rows, widths and units.

static bool wgrad_maps(const void* A1, int64_t a_cols, const void* A2, int64_t b_cols, int64_t rows, int BN,
                       GemmJob* job, CUtensorMap* mA, CUtensorMap* mB) {
  // Multi-chunk boxes need every unit's operand columns to start on a 64-column chunk and a
  // stage's BN/64 B chunks to be contiguous (one gathered group, or no gather).
  const int nbc = BN / 64;
  const bool b_contig = job->b_grp >= (1 << 29) || (job->b_grp % nbc == 0 && job->b_gs % 64 == 0);
  job->ab3d = (a_cols % 64 == 0 && b_cols % 64 == 0 && job->a_b % 64 == 0 && job->b_b % 64 == 0 && b_contig) ? 1 : 0;
  if (job->ab3d) {
    const uint64_t da[3] = {64, (uint64_t)rows, (uint64_t)a_cols / 64}, sa_[2] = {(uint64_t)a_cols * 2, 128};
    const uint64_t db[3] = {64, (uint64_t)rows, (uint64_t)b_cols / 64}, sb_[2] = {(uint64_t)b_cols * 2, 128};
    const uint32_t ba[3] = {64, 64, 2}, bb[3] = {64, 64, (uint32_t)nbc};
    if (!make_map_3d(mA, A1, da, sa_, ba, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_3d(mB, A2, db, sb_, bb, CU_TENSOR_MAP_SWIZZLE_128B))
      return false;
  } else if (!make_map_2d(mA, A1, (uint64_t)a_cols, (uint64_t)rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
             !make_map_2d(mB, A2, (uint64_t)b_cols, (uint64_t)rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) {
    return false;
  }
  job->kind = 1;
  job->rows = rows;
  job->a_cols = a_cols;
  job->b_cols = b_cols;
  job->units = (int64_t)job->mtiles * job->ntiles * job->nb * job->nsplit;
  return true;
}

template <int BN>
static cudaError_t launch_wgrad_cfg(const CUtensorMap& mA, const CUtensorMap& mB, const GemmJob& job,
                                    const CUtensorMap& mA2, const CUtensorMap& mB2, const GemmJob& job2,
                                    float* partial, int* status, cudaStream_t st, bool pdl) {
  return launch_gemm_cfg<BN, 1>(mA, mB, mA, job, mA2, mB2, job2, partial, status, st, pdl);
}

static cudaError_t launch_wgrad(int BN, const CUtensorMap& mA, const CUtensorMap& mB, const GemmJob& job,
                                const CUtensorMap& mA2, const CUtensorMap& mB2, const GemmJob& job2,
                                float* partial, int* status, cudaStream_t st, bool pdl) {
  switch (BN) {
    case 64: return launch_wgrad_cfg<64>(mA, mB, job, mA2, mB2, job2, partial, status, st, pdl);
    case 128: return launch_wgrad_cfg<128>(mA, mB, job, mA2, mB2, job2, partial, status, st, pdl);
    case 256: return launch_wgrad_cfg<256>(mA, mB, job, mA2, mB2, job2, partial, status, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t gemm_wgrad(const void* A1, int64_t a_cols, const void* A2, int64_t b_cols, int64_t rows, int BN,
                       GemmJob job, float* partial, int* status, cudaStream_t st, bool pdl) {
  CUtensorMap mA, mB;
  if (!wgrad_maps(A1, a_cols, A2, b_cols, rows, BN, &job, &mA, &mB)) return cudaErrorInvalidValue;
  const GemmJob none = {};
  return launch_wgrad(BN, mA, mB, job, mA, mB, none, partial, status, st, pdl);
}

// Operand maps of a CTA-pair job: A as (64 columns, rows, 64-column chunks) with two-chunk boxes;
// B likewise when a pair of its chunks is contiguous (ab3d = 1), else (columns, rows) with
// one-chunk boxes (ab3d = 0).  Sets kind, rows, widths; units are set by the pair launch.
static bool pair_maps(const WgradOperands& o, int64_t rows, GemmJob* job, CUtensorMap* mA, CUtensorMap* mB) {
  if (o.a_cols % 64 || job->a_b % 64) return false;
  const uint64_t da[3] = {64, (uint64_t)rows, (uint64_t)o.a_cols / 64}, sa_[2] = {(uint64_t)o.a_cols * 2, 128};
  const uint32_t box2[3] = {64, 64, 2};
  if (!make_map_3d(mA, o.A1, da, sa_, box2, CU_TENSOR_MAP_SWIZZLE_128B)) return false;
  const bool b_pairs = job->b_grp >= (1 << 29) || (job->b_grp % 2 == 0 && job->b_gs % 64 == 0);
  job->ab3d = (o.b_cols % 64 == 0 && job->b_b % 64 == 0 && b_pairs) ? 1 : 0;
  if (job->ab3d) {
    const uint64_t db[3] = {64, (uint64_t)rows, (uint64_t)o.b_cols / 64}, sb_[2] = {(uint64_t)o.b_cols * 2, 128};
    if (!make_map_3d(mB, o.A2, db, sb_, box2, CU_TENSOR_MAP_SWIZZLE_128B)) return false;
  } else if (!make_map_2d(mB, o.A2, (uint64_t)o.b_cols, (uint64_t)rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) {
    return false;
  }
  job->kind = 1;
  job->rows = rows;
  job->a_cols = o.a_cols;
  job->b_cols = o.b_cols;
  return true;
}

cudaError_t gemm_wgrad2(const WgradOperands& o1, GemmJob job1, const WgradOperands& o2, GemmJob job2,
                        int64_t rows, int BN, float* partial, int* status, cudaStream_t st, bool pdl) {
  CUtensorMap mA, mB, mA2, mB2;
  if (wgrad_pair_ok(job1, BN) && wgrad_pair_ok(job2, BN)) {
    // M tiles of 256 on CTA pairs: each CTA loads 128 columns of A and two 64-column chunks of B
    GemmJob p1 = job1, p2 = job2;
    if (pair_maps(o1, rows, &p1, &mA, &mB) && pair_maps(o2, rows, &p2, &mA2, &mB2))
      return launch_wgrad_pair(mA, mB, p1, mA2, mB2, p2, partial, status, st, pdl);
  }
  if (!wgrad_maps(o1.A1, o1.a_cols, o1.A2, o1.b_cols, rows, BN, &job1, &mA, &mB) ||
      !wgrad_maps(o2.A1, o2.a_cols, o2.A2, o2.b_cols, rows, BN, &job2, &mA2, &mB2))
    return cudaErrorInvalidValue;
  return launch_wgrad(BN, mA, mB, job1, mA2, mB2, job2, partial, status, st, pdl);
}

}  // namespace monarch
