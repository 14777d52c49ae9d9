// Fused Monarch forward for transposed outputs wider than the middle vector
// (out_transpose = 1, nb2*out2 > nb1*out1, e.g. 768 -> 3072), on tcgen05.
//
// One 64-row tile of X per unit, the whole middle vector Z on chip (shared memory).
//   1. R stage as in the row-tile kernel: M = 64 MMAs, 16 blocks per round, blocks
//      k0..k0+7 at TMEM lane offset 0 and k0+8..k0+15 at offset 16.
//   2. Permutation: 16-byte chunks of 8 consecutive k into the swizzled Z tile.
//   3. L stage in rounds of 8 output columns o: round r issues one M = 64, N = 8 MMA
//      per block j (and K step), so its result v[j][8r..8r+8) for all j is exactly the
//      contiguous output run y[r*8*nb2 .. (r+1)*8*nb2) of every row (y[o*nb2 + j]).
//   4. Each round's run is staged in its own shared-memory buffer and written with
//      TMA tensor stores of 128-byte row segments while the next round computes.
// Roles: warp 0 TMA producer (X), warp 1 MMA issuer + TMEM owner, warps 2..9 drain,
// warps 10..13 factor loaders (cp.async, see tc_rows.cu).  All waits are bounded.
#include "tc_common.cuh"

namespace monarch {

constexpr int kWideThreads = 448;
constexpr int kWideDrainWarps = 8;
constexpr int kWideLoaderThreads = 4 * 32;

template <int NB1_, int IN1_, int OUT1_, int NB2_, int IN2_, int OUT2_>
struct WideCfg {
  static constexpr int NB1 = NB1_, IN1 = IN1_, OUT1 = OUT1_, NB2 = NB2_, IN2 = IN2_, OUT2 = OUT2_;
  static constexpr int N_IN = NB1 * IN1, N_MID = NB1 * OUT1, N_OUT = NB2 * OUT2;
  static constexpr int BM = 64;
  static constexpr int KS1 = IN1 / 16, KS2 = IN2 / 16;
  static constexpr int NR1 = NB1 / 16;        // R-stage rounds of 16 blocks
  static constexpr int SLOT1 = 8 * OUT1;      // TMEM columns of one R-stage round
  static constexpr int S1_COLS = NR1 >= 2 ? 2 * SLOT1 : SLOT1;
  static constexpr int JH = NB2 / 2;          // blocks j per lane half in an L-stage round
  static constexpr int NR2 = OUT2 / 8;        // L-stage rounds of 8 output columns o
  static constexpr int SLOT2 = 8 * JH;        // TMEM columns of one L-stage round
  static constexpr int S2_COLS = 2 * SLOT2;
  static constexpr int MAXC = S1_COLS > S2_COLS ? S1_COLS : S2_COLS;
  static constexpr int TMEM_COLS = MAXC <= 64 ? 64 : (MAXC <= 128 ? 128 : (MAXC <= 256 ? 256 : 512));
  static constexpr int NXB = N_IN / 64;
  static constexpr int BPR = IN1 / 4;         // X boxes per R-stage round
  static constexpr int XBOX_BYTES = BM * 128;
  static constexpr int RPIECE = OUT1 * 32;    // R[k] rows x one 16-wide K slice (32B swizzle)
  static constexpr int STAGE_BYTES = XBOX_BYTES + 4 * RPIECE;
  static constexpr int LPIECE = 8 * 32;       // 8 rows (o) of L[j] x one 16-wide K slice
  static constexpr int LPR = NB2 * KS2;       // L slices per L-stage round
  static constexpr int LPS_MAX = STAGE_BYTES / LPIECE;
  static constexpr int LPS = LPS_MAX >= LPR ? LPR : (LPS_MAX >= LPR / 2 ? LPR / 2 : (LPS_MAX >= LPR / 3 ? LPR / 3 : LPR / 4));
  static constexpr int SPR = LPR / LPS;       // ring stages per L-stage round
  static constexpr int NSTAGE2 = NR2 * SPR;
  static constexpr int ATOM = BM * 128;
  static constexpr int ZATOMS = N_MID / 64;
  static constexpr int OW = 8 * NB2;          // output columns per L-stage round
  static constexpr int OATOMS = OW / 64;
  static constexpr int Z_BYTES = ZATOMS * ATOM, STG_BYTES = OATOMS * ATOM;
  static constexpr int NSTAGE_RAW = (kSmemBudget - Z_BYTES - STG_BYTES - 1024) / STAGE_BYTES;
  static constexpr int NSTAGE = NSTAGE_RAW > 8 ? 8 : NSTAGE_RAW;
  static constexpr int SMEM_BYTES = Z_BYTES + STG_BYTES + NSTAGE * STAGE_BYTES + 1024 + 1024;
  static constexpr int P_HALF = OUT1 / 2;

  static_assert(NB1 % 16 == 0 && NR1 <= 2, "R-stage rounds");
  static_assert(OUT1 % 16 == 0 && S1_COLS <= 512, "R-stage TMEM");
  static_assert(NB2 % 16 == 0 && OUT2 % 8 == 0, "L-stage rounds");
  static_assert(IN1 % 16 == 0 && IN2 % 16 == 0, "K steps of 16");
  static_assert(N_IN % 64 == 0 && N_MID % 64 == 0 && OW % 64 == 0, "64-column atoms");
  static_assert(NXB == NR1 * BPR, "R-stage rounds align with X boxes");
  static_assert(LPR % LPS == 0 && LPS * LPIECE <= STAGE_BYTES, "L slices per stage");
  static_assert(P_HALF % 8 == 0, "drain chunks");
  static_assert(NSTAGE >= 3, "shared memory");
};

struct WideBars {
  uint64_t full[8], empty[8];
  uint64_t a1_full[2], a2_full[2], a2_empty[2];
  uint64_t z_full, tmem_free, stg_free, staged, mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t wide_chunk_off(int r, int c) {
  const uint32_t chunk = (uint32_t)((c & 63) >> 3);
  return (uint32_t)(c >> 6) * (64 * 128) + (uint32_t)(r >> 3) * 1024 + (uint32_t)(r & 7) * 128 +
         ((chunk ^ (uint32_t)(r & 7)) << 4);
}

__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}

template <class C>
__global__ void __launch_bounds__(kWideThreads, 1)
    tc_wide_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                   const __nv_bfloat16* __restrict__ R, const __nv_bfloat16* __restrict__ L,
                   int64_t rows, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* zbuf = smem;
  uint8_t* stg = smem + C::Z_BYTES;
  uint8_t* ring = stg + C::STG_BYTES;
  WideBars* bars = (WideBars*)(ring + C::NSTAGE * C::STAGE_BYTES);
  int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t nunits = (rows + C::BM - 1) / C::BM;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      ptx::mbar_init(&bars->full[i], 1 + kWideLoaderThreads);
      ptx::mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->a1_full[i], 1);
      ptx::mbar_init(&bars->a2_full[i], 1);
      ptx::mbar_init(&bars->a2_empty[i], kWideDrainWarps);
    }
    ptx::mbar_init(&bars->z_full, kWideDrainWarps);
    ptx::mbar_init(&bars->tmem_free, kWideDrainWarps);
    ptx::mbar_init(&bars->stg_free, 1);
    ptx::mbar_init(&bars->staged, kWideDrainWarps);
    ptx::mbar_init(&bars->mma_done, 1);
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

  if (warp == 0) {
    // ================================================================ TMA producer (X)
    if (lane == 0) {
      ptx::tma_prefetch_desc(&tmX);
      ptx::tma_prefetch_desc(&tmY);
      const uint64_t pol_x = ptx::policy_evict_first();
      uint32_t it = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
        const int row0 = (int)(u * C::BM);
        for (int b = 0; b < C::NXB; ++b, ++it) {
          const int st = it % C::NSTAGE;
          if (!wait_or_abort(&bars->empty[st], ((it / C::NSTAGE) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(&bars->full[st], C::XBOX_BYTES);
          ptx::tma_load_2d(ring + st * C::STAGE_BYTES, &tmX, &bars->full[st], b * 64, row0, pol_x);
        }
        for (int sp = 0; sp < C::NSTAGE2 && ok; ++sp, ++it) {
          const int st = it % C::NSTAGE;
          if (!wait_or_abort(&bars->empty[st], ((it / C::NSTAGE) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
          ptx::mbar_arrive(&bars->full[st]);
        }
      }
      const uint32_t issued = it;
      for (uint32_t k = (issued > (uint32_t)C::NSTAGE ? issued - C::NSTAGE : 0); k < issued; ++k)
        ptx::mbar_wait_bounded(&bars->full[k % C::NSTAGE], (k / C::NSTAGE) & 1, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer (whole warp)
    constexpr uint32_t idesc1 = make_idesc(C::BM, C::OUT1);
    constexpr uint32_t idesc2 = make_idesc(C::BM, 8);
    const uint64_t ring_a = make_sdesc(ptx::smem_u32(ring), 1024, 2);
    const uint64_t ring_b = make_sdesc(ptx::smem_u32(ring), 256, 6);
    const uint64_t z_a = make_sdesc(ptx::smem_u32(zbuf), 1024, 2);
    uint32_t it = 0, rnd2 = 0, unit_n = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++unit_n) {
      // TMEM is shared by both stages: the previous unit's L-stage rounds must be drained
      if (unit_n > 0 && !warp_wait_or_abort(lane, &bars->tmem_free, (unit_n - 1) & 1, abort_flag, status)) { ok = false; break; }
      ptx::tc_fence_after();
      for (int r1 = 0; r1 < C::NR1 && ok; ++r1) {
        const uint32_t dslot = tmem + (uint32_t)(r1 * C::SLOT1);
        for (int bb = 0; bb < C::BPR; ++bb, ++it) {
          const int st = it % C::NSTAGE;
          if (!warp_wait_or_abort(lane, &bars->full[st], (it / C::NSTAGE) & 1, abort_flag, status)) { ok = false; break; }
          ptx::fence_proxy_async_smem();
          ptx::tc_fence_after();
          const uint64_t soff = (uint64_t)((st * C::STAGE_BYTES) >> 4);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int c = bb * 64 + 16 * t;
            const int kk = c / C::IN1, s16 = (c % C::IN1) / 16;
            const uint32_t d = dslot + ((uint32_t)(kk >> 3) << 20) + (uint32_t)((kk & 7) * C::OUT1);
            ptx::mma_bf16_ss_elect(d, ring_a + soff + (uint64_t)((32 * t) >> 4),
                                   ring_b + soff + (uint64_t)((C::XBOX_BYTES + t * C::RPIECE) >> 4),
                                   idesc1, s16 > 0 ? 1u : 0u);
          }
          ptx::mma_commit_elect(&bars->empty[st]);
        }
        if (!ok) break;
        ptx::mma_commit_elect(&bars->a1_full[r1]);
      }
      if (!ok) break;
      if (!warp_wait_or_abort(lane, &bars->z_full, unit_n & 1, abort_flag, status)) { ok = false; break; }
      ptx::tc_fence_after();
      for (int r2 = 0; r2 < C::NR2 && ok; ++r2, ++rnd2) {
        const int slot = rnd2 & 1;
        if (!warp_wait_or_abort(lane, &bars->a2_empty[slot], ((rnd2 >> 1) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t dslot = tmem + (uint32_t)(slot * C::SLOT2);
        for (int sp = 0; sp < C::SPR; ++sp, ++it) {
          const int st = it % C::NSTAGE;
          if (!warp_wait_or_abort(lane, &bars->full[st], (it / C::NSTAGE) & 1, abort_flag, status)) { ok = false; break; }
          ptx::fence_proxy_async_smem();
          ptx::tc_fence_after();
          const uint64_t soff = (uint64_t)((st * C::STAGE_BYTES) >> 4);
#pragma unroll 4
          for (int t = 0; t < C::LPS; ++t) {
            const int piece = sp * C::LPS + t;  // within the round: j * KS2 + s
            const int j = piece / C::KS2, s16 = piece % C::KS2;
            const int h = j / C::JH, jj = j % C::JH;
            const int zc = j * C::IN2 + 16 * s16;
            const uint32_t d = dslot + ((uint32_t)h << 20) + (uint32_t)(jj * 8);
            ptx::mma_bf16_ss_elect(d, z_a + (uint64_t)(((zc >> 6) * C::ATOM + (zc & 63) * 2) >> 4),
                                   ring_b + soff + (uint64_t)((t * C::LPIECE) >> 4), idesc2,
                                   s16 > 0 ? 1u : 0u);
          }
          ptx::mma_commit_elect(&bars->empty[st]);
        }
        if (!ok) break;
        ptx::mma_commit_elect(&bars->a2_full[slot]);
      }
    }
    ptx::mma_commit_elect(&bars->mma_done);
    if (lane == 0) ptx::mbar_wait_bounded(&bars->mma_done, 0, kWaitLimitNs);
    __syncwarp();
  } else if (warp >= 2 + kWideDrainWarps) {
    // ================================================================ factor loaders
    const int lt = (warp - 2 - kWideDrainWarps) * 32 + lane;
    const uint32_t ring_s = ptx::smem_u32(ring);
    uint32_t it = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
      for (int sq = 0; sq < C::NXB + C::NSTAGE2 && ok; ++sq, ++it) {
        const int st = it % C::NSTAGE;
        if (!wait_or_abort(&bars->empty[st], ((it / C::NSTAGE) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
        const uint32_t sb = ring_s + st * C::STAGE_BYTES;
        if (sq < C::NXB) {
          const int b = sq;
          for (int g = lt; g < 4 * C::OUT1 * 2; g += kWideLoaderThreads) {
            const int t = g / (C::OUT1 * 2), n = (g >> 1) % C::OUT1, c = g & 1;
            const int col = b * 64 + t * 16;
            const int k = col / C::IN1, s16 = col % C::IN1;
            ptx::cp_async_16(sb + C::XBOX_BYTES + t * C::RPIECE + n * 32 + ((c ^ ((n >> 2) & 1)) << 4),
                             R + ((int64_t)k * C::OUT1 + n) * C::IN1 + s16 + c * 8);
          }
        } else {
          const int q = sq - C::NXB;
          const int r2 = q / C::SPR, sp = q % C::SPR;
          for (int g = lt; g < C::LPS * 16; g += kWideLoaderThreads) {  // 8 rows x 2 chunks per slice
            const int t = g / 16, n = (g >> 1) & 7, c = g & 1;
            const int piece = sp * C::LPS + t, j = piece / C::KS2, s16 = (piece % C::KS2) * 16;
            ptx::cp_async_16(sb + t * C::LPIECE + n * 32 + ((c ^ ((n >> 2) & 1)) << 4),
                             L + ((int64_t)j * C::OUT2 + r2 * 8 + n) * C::IN2 + s16 + c * 8);
          }
        }
        ptx::cp_async_mbar_arrive_noinc(&bars->full[st]);
      }
    }
    ptx::cp_async_wait<0>();
  } else {
    // ================================================================ drain (8 warps)
    const int quad = warp & 3, ph = (warp - 2) >> 2, half = lane >> 4;
    const int r = quad * 16 + (lane & 15);
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t z_s = ptx::smem_u32(zbuf), stg_s = ptx::smem_u32(stg);
    const bool leader = (warp == 2 && lane == 0);
    uint32_t rnd2 = 0, unit_n = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++unit_n) {
      for (int r1 = 0; r1 < C::NR1 && ok; ++r1) {
        if (!wait_or_abort(&bars->a1_full[r1], unit_n & 1, abort_flag, status)) { ok = false; break; }
        __syncwarp();  // the leader lane may still be coming out of the previous unit's store branch
        ptx::tc_fence_after();
        const uint32_t tb = tmem + lane_off + (uint32_t)(r1 * C::SLOT1);
#pragma unroll 1
        for (int pc = ph * C::P_HALF; pc < (ph + 1) * C::P_HALF; pc += 8) {
          float v[8][8];
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            uint32_t rr[8];
            ptx::tmem_ld8(tb + kk * C::OUT1 + pc, rr);
#pragma unroll
            for (int e = 0; e < 8; ++e) v[kk][e] = __uint_as_float(rr[e]);
          }
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int t0 = (pc + e) * C::NB1 + r1 * 16 + half * 8;
            ptx::st_shared_v4(z_s + wide_chunk_off(r, t0), ptx::pack_bf16x2(v[0][e], v[1][e]),
                              ptx::pack_bf16x2(v[2][e], v[3][e]), ptx::pack_bf16x2(v[4][e], v[5][e]),
                              ptx::pack_bf16x2(v[6][e], v[7][e]));
          }
        }
      }
      if (!ok) break;
      ptx::tc_fence_before();
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->z_full);
      const int row0 = (int)(u * C::BM);
      for (int r2 = 0; r2 < C::NR2 && ok; ++r2, ++rnd2) {
        const int slot = rnd2 & 1;
        if (!wait_or_abort(&bars->a2_full[slot], (rnd2 >> 1) & 1, abort_flag, status)) { ok = false; break; }
        // the staging buffer must have been read out by the previous round's stores
        if (leader) {
          ptx::bulk_wait_read_all();
          ptx::mbar_arrive(&bars->stg_free);
        }
        if (!wait_or_abort(&bars->stg_free, rnd2 & 1, abort_flag, status)) { ok = false; break; }
        __syncwarp();  // tcgen05.ld is warp-collective
        ptx::tc_fence_after();
        const uint32_t tb = tmem + lane_off + (uint32_t)(slot * C::SLOT2);
#pragma unroll 1
        for (int jc = 0; jc < C::JH / 8; ++jc) {
          float v[8][4];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            uint32_t rr[4];
            tmem_ld4(tb + (jc * 8 + jj) * 8 + 4 * ph, rr);
#pragma unroll
            for (int e = 0; e < 4; ++e) v[jj][e] = __uint_as_float(rr[e]);
          }
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 4; ++e) {  // local column (o - 8 r2) * nb2 + j, 8 consecutive j
            const int lc = (4 * ph + e) * C::NB2 + half * C::JH + jc * 8;
            ptx::st_shared_v4(stg_s + wide_chunk_off(r, lc), ptx::pack_bf16x2(v[0][e], v[1][e]),
                              ptx::pack_bf16x2(v[2][e], v[3][e]), ptx::pack_bf16x2(v[4][e], v[5][e]),
                              ptx::pack_bf16x2(v[6][e], v[7][e]));
          }
        }
        ptx::tc_fence_before();
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive(&bars->a2_empty[slot]);
          ptx::mbar_arrive(&bars->staged);
        }
        if (leader) {
          if (!wait_or_abort(&bars->staged, rnd2 & 1, abort_flag, status)) {
            ok = false;
          } else {
            for (int a = 0; a < C::OATOMS; ++a)
              ptx::tma_store_2d(&tmY, stg + a * C::ATOM, r2 * C::OW + a * 64, row0);
            ptx::bulk_commit_group();
          }
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->tmem_free);
    }
    if (leader) ptx::bulk_wait_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

template <class C>
static cudaError_t launch_wide(const void* X, const void* R, const void* L, void* Y, int64_t rows,
                               int* status, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  CUtensorMap mX, mY;
  if (!make_map_2d(&mX, X, C::N_IN, (uint64_t)rows, 64, C::BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mY, Y, C::N_OUT, (uint64_t)rows, 64, C::BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(tc_wide_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int64_t nunits = (rows + C::BM - 1) / C::BM;
  int64_t grid = num_sms();
  if (grid > nunits) grid = nunits;
  tc_wide_kernel<C><<<(unsigned)grid, kWideThreads, C::SMEM_BYTES, st>>>(
      mX, mY, (const __nv_bfloat16*)R, (const __nv_bfloat16*)L, rows, status);
  return cudaGetLastError();
}

using WideR768 = WideCfg<16, 48, 48, 48, 16, 64>;  // 768 -> 3072

template <class C>
static bool wide_shape_is(const Shape& s) {
  return s.nb1 == C::NB1 && s.in1 == C::IN1 && s.out1 == C::OUT1 && s.nb2 == C::NB2 &&
         s.in2 == C::IN2 && s.out2 == C::OUT2 && s.out_transpose == 1;
}

bool tc_wide_supported(const Shape& s) { return wide_shape_is<WideR768>(s); }

cudaError_t tc_wide_fwd(const void* X, const void* R, const void* L, void* Y, const Shape& s,
                        int* status, cudaStream_t st) {
  if (wide_shape_is<WideR768>(s)) return launch_wide<WideR768>(X, R, L, Y, s.rows, status, st);
  return cudaErrorNotSupported;
}

}  // namespace monarch
