// tcgen05 GEMMs on CTA pairs (two-CTA clusters, cta_group::2): one M = 256, N = 256 MMA tile per
// pair, each CTA loading half of A and half of B into the same shared-memory offsets and receiving
// its 128 rows of D in its own TMEM.  Per K stage each SM then holds 32 KB for a 128 x 256 x 64
// share of the product (against 48 KB for the same work on one CTA), so more stages fit.
//
// tc_wgrad_pair_kernel: the weight gradient (tc_gemm_kernel kind 1 jobs with M tiles of 256:
//   D[m][n] = sum_rows act1[r][m] * act2[r][n], fp32 partials of the diagonal blocks), for block
//   groups of 256 or more rows on the M side (e.g. nblocks = 4: dR over 256 x 256 blocks, dL over
//   1024 x 256 blocks).  CTA r of the pair loads A columns [mt*256 + 128 r, +128) and B chunks
//   2r, 2r + 1 of the unit's four 64-column chunks (gathered like kind 1's), K = 64 rows a stage.
// tc_bd_pair_kernel: the block-diagonal stage with streamed weights (tc_gemm_kernel kind 0 jobs with
//   BN = 256 and M tiles of 256 rows), Y = A W^T per block: CTA r loads A rows
//   [mt*256 + 128 r, +128) and W rows [nt*256 + 128 r, +128) of the block, K = 64 a stage, and
//   writes its 128 output rows with TMA stores.
//
// Synchronisation (both CTAs lay out the same barriers at the same offsets):
//   full[s]      first CTA only: its producer arrives with the transaction bytes of both CTAs'
//                loads; both CTAs' TMA loads complete on it.
//   empty[s]     both CTAs: the pair MMA's commit arrives on both (multicast).
//   acc_full[k]  both CTAs: the pair MMA's commit after a unit's last K stage.
//   acc_empty[k] first CTA only: the epilogue warps of both CTAs arrive (the second CTA's remotely).
//   mma_done     both CTAs: the final commit.
// All mbarrier waits are bounded; a cluster barrier after setup and before teardown keeps
// either CTA from touching the other's barriers or shared memory before they exist or after it
// has left.
#include "tc_common.cuh"
#include "tc_gemm.cuh"

namespace monarch {

constexpr int kPairThreads = 192;
constexpr int kPairEpiWarps = 4;

struct PairCfg {
  static constexpr int BM = 128;                 // D rows per CTA (M = 256 per pair)
  static constexpr int BN = 256;                 // D columns (N per pair)
  static constexpr int A_BYTES = BM * 128;       // 128 M indices x 64 rows (MN-major, two 64-wide atoms)
  static constexpr int B_BYTES = (BN / 2) * 128; // this CTA's 128 N indices x 64 rows
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int NSTAGE_RAW = (kSmemBudget - 1024) / STAGE;
  static constexpr int NSTAGE = NSTAGE_RAW > 8 ? 8 : NSTAGE_RAW;
  static constexpr int SMEM_BYTES = NSTAGE * STAGE + 1024 + 1024;
  static constexpr int TMEM_COLS = 2 * BN;       // two accumulator slots of 256 columns
  static_assert(NSTAGE >= 4, "shared memory");
};

struct PairBars {
  uint64_t full[8], empty[8];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

struct PairUnit {
  int b, mt, split, second;
};

// Unit u of the launch (the second job's units follow the first's); the unit order inside a job
// is m tile, group, split (n tile count is 1: N = 256 covers the group's columns).
__device__ __forceinline__ PairUnit pair_unit(const GemmJob& j1, const GemmJob& j2, int64_t u) {
  const bool second = u >= j1.units;
  const GemmJob& j = second ? j2 : j1;
  if (second) u -= j1.units;
  PairUnit c;
  c.mt = (int)(u % j.mtiles);
  u /= j.mtiles;
  c.b = (int)(u % j.nb);
  c.split = (int)(u / j.nb);
  c.second = second ? 1 : 0;
  return c;
}

__device__ __forceinline__ int pair_kstages(const GemmJob& j, const PairUnit& c) {
  int64_t n = j.rows - (int64_t)c.split * j.split_rows;
  if (n > j.split_rows) n = j.split_rows;
  return (int)((n + 63) / 64);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    tc_wgrad_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ GemmJob job, const __grid_constant__ CUtensorMap tmA2,
                         const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ GemmJob job2,
                         float* __restrict__ partial, int* status) {
  using C = PairCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = smem;
  PairBars* bars = (PairBars*)(ring + C::NSTAGE * C::STAGE);
  int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool first = rank == 0;
  const int64_t cl = blockIdx.x / 2, ncl = gridDim.x / 2;
  const int64_t total = job.units + job2.units;
  const int64_t nmine = total > cl ? (total - cl + ncl - 1) / ncl : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      ptx::mbar_init(&bars->full[i], 1);
      ptx::mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->acc_full[i], 1);
      ptx::mbar_init(&bars->acc_empty[i], 2 * kPairEpiWarps);
    }
    ptx::mbar_init(&bars->mma_done, 1);
    bars->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(&bars->tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  if (warp == 0) {
    // ================================================================ TMA producer (both CTAs)
    if (lane == 0) {
      ptx::tma_prefetch_desc(&tmA);
      ptx::tma_prefetch_desc(&tmB);
      if (job2.units > 0) {
        ptx::tma_prefetch_desc(&tmA2);
        ptx::tma_prefetch_desc(&tmB2);
      }
      const uint64_t pol = ptx::policy_evict_normal();
      const uint32_t full0 = ptx::mapa_shared(ptx::smem_u32(&bars->full[0]), 0);  // first CTA's full[0]
      uint32_t it = 0;
      bool ok = true;
      for (int64_t i = 0; i < nmine && ok; ++i) {
        const PairUnit c = pair_unit(job, job2, cl + i * ncl);
        const GemmJob& jb = c.second ? job2 : job;
        const CUtensorMap* mapA = c.second ? &tmA2 : &tmA;
        const CUtensorMap* mapB = c.second ? &tmB2 : &tmB;
        const int nk = pair_kstages(jb, c);
        const int ax = c.b * jb.a_b + c.mt * 256 + (int)rank * 128;
        const int bx = gcol(c.b, jb.b_b, 2 * (int)rank, jb.b_grp, jb.b_gs);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int st = it % C::NSTAGE;
          if (!wait_or_abort(&bars->empty[st], ((it / C::NSTAGE) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
          uint8_t* sa = ring + st * C::STAGE;
          const int row = (int)((int64_t)c.split * jb.split_rows + (int64_t)kb * 64);
          if (first) ptx::mbar_arrive_expect_tx(&bars->full[st], 2 * C::STAGE);
          const uint32_t fb = full0 + (uint32_t)(st * sizeof(uint64_t));
          ptx::tma_load_3d_pair(sa, mapA, fb, 0, row, ax / 64, pol);
          if (jb.ab3d) {
            ptx::tma_load_3d_pair(sa + C::A_BYTES, mapB, fb, 0, row, bx / 64, pol);
          } else {  // the two B chunks are gathered from separate column groups
            ptx::tma_load_2d_pair(sa + C::A_BYTES, mapB, fb, bx, row, pol);
            ptx::tma_load_2d_pair(sa + C::A_BYTES + 8192, mapB, fb,
                                  gcol(c.b, jb.b_b, 2 * (int)rank + 1, jb.b_grp, jb.b_gs), row, pol);
          }
        }
      }
      // the loads of the last stages land before the pair's MMAs complete; the teardown waits
      // for those (mma_done) before either CTA leaves
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer (first CTA)
    if (first) {
      constexpr uint32_t idesc = make_idesc(256, C::BN) | (1u << 15) | (1u << 16);  // A, B MN-major
      const uint64_t dA = make_sdesc_lbo(ptx::smem_u32(ring), 8192, 1024, 2);
      const uint64_t dB = make_sdesc_lbo(ptx::smem_u32(ring + C::A_BYTES), 8192, 1024, 2);
      constexpr uint64_t kstep = 2048 >> 4;  // 16 rows of K: two 8-row groups of 1024 B
      uint32_t it = 0, n = 0;
      bool ok = true;
      for (int64_t i = 0; i < nmine && ok; ++i, ++n) {
        const PairUnit c = pair_unit(job, job2, cl + i * ncl);
        const int nk = pair_kstages(c.second ? job2 : job, c);
        const int slot = n & 1;
        if (!warp_wait_or_abort(lane, &bars->acc_empty[slot], ((n >> 1) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t d = tmem + slot * C::BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int st = it % C::NSTAGE;
          if (!warp_wait_or_abort(lane, &bars->full[st], (it / C::NSTAGE) & 1, abort_flag, status)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint64_t soff = (uint64_t)((st * C::STAGE) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_bf16_ss_pair_elect(d, dA + soff + kk * kstep, dB + soff + kk * kstep, idesc,
                                        (kb > 0 || kk > 0) ? 1u : 0u);
          ptx::mma_commit_pair_elect(&bars->empty[st], 0x3);  // both CTAs may refill the stage
        }
        if (!ok) break;
        ptx::mma_commit_pair_elect(&bars->acc_full[slot], 0x3);
      }
      ptx::mma_commit_pair_elect(&bars->mma_done, 0x3);
    }
    // both CTAs: every pair MMA (which reads both CTAs' shared memory) has completed
    if (lane == 0) wait_mma_done(&bars->mma_done, abort_flag, status);
    __syncwarp();
  } else {
    // ================================================================ epilogue (4 warps, both CTAs)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // D row of this thread within this CTA's 128
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t acc_empty0 = ptx::mapa_shared(ptx::smem_u32(&bars->acc_empty[0]), 0);
    uint32_t n = 0;
    bool ok = true;
    for (int64_t i = 0; i < nmine && ok; ++i, ++n) {
      const PairUnit c = pair_unit(job, job2, cl + i * ncl);
      const GemmJob& jb = c.second ? job2 : job;
      const int slot = n & 1;
      if (!wait_or_abort(&bars->acc_full[slot], (n >> 1) & 1, abort_flag, status)) { ok = false; break; }
      ptx::tc_fence_after();
      const uint32_t tb = tmem + lane_off + slot * C::BN;
      // diagonal blocks of D as fp32 partials, as in tc_gemm_kernel kind 1
      const int bla = (int)jb.blk_a, blb = (int)jb.blk_b;
      const int mrow0 = c.b * jb.a_b + c.mt * 256 + (int)rank * 128;
      const int ma = mrow0 + r;
      const int nb0 = c.b * jb.b_lb;
      const int blk = ma / bla;
      const bool row_ok = ma < (int)jb.a_cols;
      const int t_lo = max(0, blk * blb - nb0);
      const int t_hi = min(C::BN, min((blk + 1) * blb, (int)jb.b_cols) - nb0);
      const int ma0 = mrow0 + quad * 32;
      const int w_lo = max(0, (ma0 / bla) * blb - nb0) & ~15;
      const int w_hi = min(C::BN, ((ma0 + 31) / bla + 1) * blb - nb0);
      float* prow = partial + (int64_t)c.split * jb.p_stride + jb.p_off + (int64_t)blk * bla * blb +
                    (int64_t)(ma - blk * bla) * blb + (nb0 - blk * blb);
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
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (first)
          ptx::mbar_arrive(&bars->acc_empty[slot]);
        else
          ptx::mbar_arrive_cluster(acc_empty0 + (uint32_t)(slot * sizeof(uint64_t)));
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync_all();  // neither CTA leaves while the pair's MMAs or the peer may use it
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc_pair(tmem, C::TMEM_COLS);
}

bool wgrad_pair_ok(const GemmJob& j, int BN) {
  return BN == 256 && j.a_b % 256 == 0 && j.mtiles % 2 == 0 && j.ntiles == 1;
}

cudaError_t launch_wgrad_pair(const CUtensorMap& mA, const CUtensorMap& mB, GemmJob job, const CUtensorMap& mA2,
                              const CUtensorMap& mB2, GemmJob job2, float* partial, int* status, cudaStream_t st,
                              bool pdl) {
  using C = PairCfg;
  cudaError_t e = ensure_smem_attr((const void*)tc_wgrad_pair_kernel, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  job.mtiles /= 2;  // M tiles of 256 rows
  job.units = (int64_t)job.mtiles * job.nb * job.nsplit;
  job2.mtiles /= 2;
  job2.units = (int64_t)job2.mtiles * job2.nb * job2.nsplit;
  int64_t pairs = num_sms() / 2;
  const int64_t units = job.units + job2.units;
  if (pairs > units) pairs = units;
  return launch_kernel(tc_wgrad_pair_kernel, dim3((unsigned)(2 * pairs)), dim3(kPairThreads), C::SMEM_BYTES, st, pdl,
                       mA, mB, job, mA2, mB2, job2, partial, status);
}


// ---------------------------------------------------------------- block-diagonal stage on pairs
struct PairBdCfg {
  static constexpr int BM = 128;                 // output rows per CTA (M = 256 per pair)
  static constexpr int BN = 256;                 // output columns per unit
  static constexpr int A_BYTES = BM * 128;       // 128 rows x 64 K (K-major, 128B swizzle)
  static constexpr int B_BYTES = (BN / 2) * 128; // this CTA's 128 weight rows x 64 K
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STG_BYTES = 2 * BM * 128; // two 128 x 64 output chunks
  static constexpr int NSTAGE_RAW = (kSmemBudget - STG_BYTES - 1024) / STAGE;
  static constexpr int NSTAGE = NSTAGE_RAW > 8 ? 8 : NSTAGE_RAW;
  static constexpr int SMEM_BYTES = STG_BYTES + NSTAGE * STAGE + 1024 + 1024;
  static constexpr int TMEM_COLS = 2 * BN;
  static_assert(NSTAGE >= 4, "shared memory");
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    tc_bd_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmY, const __grid_constant__ GemmJob job, int* status) {
  using C = PairBdCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stg = smem;                 // two output staging chunks
  uint8_t* ring = smem + C::STG_BYTES;
  PairBars* bars = (PairBars*)(ring + C::NSTAGE * C::STAGE);
  int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool first = rank == 0;
  const int64_t cl = blockIdx.x / 2, ncl = gridDim.x / 2;
  const int64_t nmine = job.units > cl ? (job.units - cl + ncl - 1) / ncl : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      ptx::mbar_init(&bars->full[i], 1);
      ptx::mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->acc_full[i], 1);
      ptx::mbar_init(&bars->acc_empty[i], 2 * kPairEpiWarps);
    }
    ptx::mbar_init(&bars->mma_done, 1);
    bars->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(&bars->tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  // unit u: n tile fastest, then block, then 256-row m tile
  auto unit = [&](int64_t u, int* b, int* mt, int* nt) {
    *nt = (int)(u % job.ntiles);
    u /= job.ntiles;
    *b = (int)(u % job.nb);
    *mt = (int)(u / job.nb);
  };

  if (warp == 0) {
    // ================================================================ TMA producer (both CTAs)
    if (lane == 0) {
      ptx::tma_prefetch_desc(&tmA);
      ptx::tma_prefetch_desc(&tmB);
      ptx::tma_prefetch_desc(&tmY);
      const uint64_t pol = ptx::policy_evict_normal();
      const uint32_t full0 = ptx::mapa_shared(ptx::smem_u32(&bars->full[0]), 0);
      uint32_t it = 0;
      bool ok = true;
      for (int64_t i = 0; i < nmine && ok; ++i) {
        int b, mt, nt;
        unit(cl + i * ncl, &b, &mt, &nt);
        const int arow = mt * 256 + (int)rank * 128;
        const int wrow = b * job.b_b + nt * C::BN + (int)rank * 128;
        for (int kb = 0; kb < job.kboxes; ++kb, ++it) {
          const int st = it % C::NSTAGE;
          if (!wait_or_abort(&bars->empty[st], ((it / C::NSTAGE) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
          uint8_t* sa = ring + st * C::STAGE;
          if (first) ptx::mbar_arrive_expect_tx(&bars->full[st], 2 * C::STAGE);
          const uint32_t fb = full0 + (uint32_t)(st * sizeof(uint64_t));
          ptx::tma_load_2d_pair(sa, &tmA, fb, gcol(b, job.a_b, kb, job.a_grp, job.a_gs), arow, pol);
          ptx::tma_load_2d_pair(sa + C::A_BYTES, &tmB, fb, kb * 64, wrow, pol);
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer (first CTA)
    if (first) {
      constexpr uint32_t idesc = make_idesc(256, C::BN);  // A, B K-major
      const uint64_t dA = make_sdesc(ptx::smem_u32(ring), 1024, 2);
      const uint64_t dB = make_sdesc(ptx::smem_u32(ring + C::A_BYTES), 1024, 2);
      constexpr uint64_t kstep = 32 >> 4;  // 16 K values: 32 bytes of a swizzled 128-byte row
      uint32_t it = 0, n = 0;
      bool ok = true;
      for (int64_t i = 0; i < nmine && ok; ++i, ++n) {
        const int slot = n & 1;
        if (!warp_wait_or_abort(lane, &bars->acc_empty[slot], ((n >> 1) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t d = tmem + slot * C::BN;
        for (int kb = 0; kb < job.kboxes; ++kb, ++it) {
          const int st = it % C::NSTAGE;
          if (!warp_wait_or_abort(lane, &bars->full[st], (it / C::NSTAGE) & 1, abort_flag, status)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint64_t soff = (uint64_t)((st * C::STAGE) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_bf16_ss_pair_elect(d, dA + soff + kk * kstep, dB + soff + kk * kstep, idesc,
                                        (kb > 0 || kk > 0) ? 1u : 0u);
          ptx::mma_commit_pair_elect(&bars->empty[st], 0x3);
        }
        if (!ok) break;
        ptx::mma_commit_pair_elect(&bars->acc_full[slot], 0x3);
      }
      ptx::mma_commit_pair_elect(&bars->mma_done, 0x3);
    }
    if (lane == 0) wait_mma_done(&bars->mma_done, abort_flag, status);
    __syncwarp();
  } else {
    // ================================================================ epilogue (4 warps, both CTAs)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // output row of this thread within this CTA's 128
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool leader = (warp == 2 && lane == 0);
    const uint32_t stg_s = ptx::smem_u32(stg);
    const uint32_t acc_empty0 = ptx::mapa_shared(ptx::smem_u32(&bars->acc_empty[0]), 0);
    uint32_t n = 0, chunk_n = 0;
    bool ok = true;
    for (int64_t i = 0; i < nmine && ok; ++i, ++n) {
      int b, mt, nt;
      unit(cl + i * ncl, &b, &mt, &nt);
      const int slot = n & 1;
      if (!wait_or_abort(&bars->acc_full[slot], (n >> 1) & 1, abort_flag, status)) { ok = false; break; }
      ptx::tc_fence_after();
      const uint32_t tb = tmem + lane_off + slot * C::BN;
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
        ptx::named_bar_sync(1, kPairEpiWarps * 32);
        const uint32_t base = stg_s + sbuf * (C::BM * 128) + r * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          ptx::st_shared_v4(base + (((uint32_t)q ^ (uint32_t)(r & 7)) << 4),
                            ptx::pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1])),
                            ptx::pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                            ptx::pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                            ptx::pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
        ptx::fence_proxy_async_smem();
        ptx::named_bar_sync(1, kPairEpiWarps * 32);
        if (leader) {
          ptx::tma_store_2d(&tmY, stg + sbuf * (C::BM * 128),
                            gcol(b, job.y_b, nt * (C::BN / 64) + ch, job.y_grp, job.y_gs), mt * 256 + (int)rank * 128);
          ptx::bulk_commit_group();
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (first)
          ptx::mbar_arrive(&bars->acc_empty[slot]);
        else
          ptx::mbar_arrive_cluster(acc_empty0 + (uint32_t)(slot * sizeof(uint64_t)));
      }
    }
    if (leader) ptx::bulk_wait_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync_all();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc_pair(tmem, C::TMEM_COLS);
}

cudaError_t gemm_bd_pair(const void* A, int64_t rows, int64_t a_cols, const void* W, int64_t w_rows, int K, void* Y,
                         int64_t y_cols, GemmJob job, int* status, cudaStream_t st, bool pdl) {
  using C = PairBdCfg;
  CUtensorMap mA, mB, mY;
  if (!make_map_2d(&mA, A, (uint64_t)a_cols, (uint64_t)rows, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mB, W, (uint64_t)K, (uint64_t)w_rows, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mY, Y, (uint64_t)y_cols, (uint64_t)rows, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_attr((const void*)tc_bd_pair_kernel, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  job.kind = 0;
  job.mtiles = (int)((rows + 255) / 256);  // M tiles of 256 rows
  job.units = (int64_t)job.mtiles * job.nb * job.ntiles;
  int64_t pairs = num_sms() / 2;
  if (pairs > job.units) pairs = job.units;
  return launch_kernel(tc_bd_pair_kernel, dim3((unsigned)(2 * pairs)), dim3(kPairThreads), C::SMEM_BYTES, st, pdl,
                       mA, mB, mY, job, status);
}

}  // namespace monarch
