// Fused Monarch forward for transposed outputs wider than the middle vector
// (out_transpose = 1, nb2*out2 > nb1*out1 and nb1*in1 <= nb1*out1, e.g. 768 -> 3072), on
// tcgen05.  One tile of bm <= 64 rows of X per unit, the whole middle vector on chip.
//
//   1. The whole X tile is loaded by TMA straight into the buffer that later holds the
//      middle tile Z (128B-swizzled 64-column atoms), and all of R into the output
//      staging area (idle until the L stage), so the R stage has no ring to wait on.
//      R stage: M = 64 MMAs, blocks k0..k0+7 at TMEM lane offset 0 and k0+8..k0+15 at
//      lane offset 16.
//   2. Permutation: the drain warps write 16-byte chunks of 8 consecutive k into Z,
//      over the (now consumed) X tile.
//   3. L stage in rounds of 8 output columns o: round r issues one M = 64, N = 8 MMA per
//      block j, so its result v[j][8r..8r+8) for all j is the contiguous output run
//      y[r*8*nb2 .. (r+1)*8*nb2) of every row (y[o*nb2 + j]).  The L slices of a round
//      come through a two-stage ring.
//   4. Each round's run is staged in one of two shared-memory buffers and written with
//      TMA tensor stores while the next round computes and drains into the other.
// With SAVE, the middle tile Z (the L stage's input vector, bf16) is also written to global
// memory with TMA stores as soon as the drain has built it (the training forward keeps it for
// the backward).
// bm (rows per unit, a multiple of 8) is chosen on the host so the units spread evenly
// over the SMs; MMAs always cover 64 rows, and rows >= bm of a tile are never stored.
// Roles: warp 0 TMA producer (X), warp 1 MMA issuer + TMEM owner, warps 2..9 drain,
// warps 10..13 factor loaders (16-byte cp.async, software 32B swizzle).  All waits are
// bounded (tc_common.cuh).
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
  static constexpr int KS2 = IN2 / 16;
  static constexpr int SLOT1 = 8 * OUT1;      // TMEM columns of the R stage (16 blocks)
  static constexpr int JH = NB2 / 2;          // blocks j per lane half in an L-stage round
  static constexpr int NR2 = OUT2 / 8;        // L-stage rounds of 8 output columns o
  static constexpr int SLOT2 = 8 * JH;        // TMEM columns of one L-stage round
  static constexpr int MAXC = SLOT1 > 2 * SLOT2 ? SLOT1 : 2 * SLOT2;
  static constexpr int TMEM_COLS = MAXC <= 128 ? 128 : (MAXC <= 256 ? 256 : 512);
  static constexpr int NXB = N_IN / 64;       // X boxes (64 columns) per tile
  static constexpr int ATOM = BM * 128;       // 64 rows x 64 bf16 columns, 128B swizzle
  static constexpr int RPIECE = OUT1 * 32;    // R[k] rows x one 16-wide K slice, 32B swizzle
  static constexpr int NRP = N_IN / 16;       // R slices (k, s) = column slice / 16
  static constexpr int LPIECE = 8 * 32;       // 8 rows (o) of L[j] x one 16-wide K slice
  static constexpr int LPR = NB2 * KS2;       // L slices per round
  static constexpr int LSTAGE = LPR * LPIECE;
  static constexpr int ZATOMS = N_MID / 64;
  static constexpr int OW = 8 * NB2;          // output columns per round
  static constexpr int OATOMS = OW / 64;
  static constexpr int Z_BYTES = ZATOMS * ATOM, STG_BYTES = OATOMS * ATOM;
  static constexpr int SMEM_BYTES = Z_BYTES + 2 * STG_BYTES + 2 * LSTAGE + 1024 + 1024;
  static constexpr int P_HALF = OUT1 / 2;

  static_assert(NB1 == 16, "one R-stage round of 16 blocks");
  static_assert(OUT1 % 16 == 0 && SLOT1 <= 512, "R-stage TMEM");
  static_assert(NB2 % 16 == 0 && OUT2 % 8 == 0 && JH % 8 == 0, "L-stage rounds");
  static_assert(IN1 % 16 == 0 && IN2 % 16 == 0, "K steps of 16");
  static_assert(N_IN % 64 == 0 && N_MID % 64 == 0 && OW % 64 == 0, "64-column atoms");
  static_assert(N_IN <= N_MID, "the X tile is loaded into the middle-tile buffer");
  static_assert(NRP * RPIECE <= 2 * STG_BYTES, "R is parked in the staging buffers");
  static_assert(NXB <= 16, "X box barriers");
  static_assert(P_HALF % 8 == 0, "drain chunks");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct WideBars {
  uint64_t xfull[16];            // X box b and its four R slices (TMA bytes + loader arrivals)
  uint64_t lfull[2], lempty[2];  // L ring
  uint64_t a1_full, a2_full[2], a2_empty[2];
  uint64_t z_full, tmem_free, rfree, stg_free, staged, mma_done;
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

template <class C, int SAVE>
__global__ void __launch_bounds__(kWideThreads, 1)
    tc_wide_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                   const __grid_constant__ CUtensorMap tmZ, const __nv_bfloat16* __restrict__ R,
                   const __nv_bfloat16* __restrict__ L, int64_t rows, int bm, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* zbuf = smem;                    // X tile, then Z tile
  uint8_t* stg = smem + C::Z_BYTES;        // R during the R stage, then 2 output buffers
  uint8_t* ring = stg + 2 * C::STG_BYTES;  // 2 L stages
  WideBars* bars = (WideBars*)(ring + 2 * C::LSTAGE);
  int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t nunits = (rows + bm - 1) / bm;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NXB; ++i) ptx::mbar_init(&bars->xfull[i], 1 + kWideLoaderThreads);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->lfull[i], kWideLoaderThreads);
      ptx::mbar_init(&bars->lempty[i], 1);
      ptx::mbar_init(&bars->a2_full[i], 1);
      ptx::mbar_init(&bars->a2_empty[i], kWideDrainWarps);
    }
    ptx::mbar_init(&bars->a1_full, 1);
    ptx::mbar_init(&bars->z_full, kWideDrainWarps);
    ptx::mbar_init(&bars->tmem_free, kWideDrainWarps);
    ptx::mbar_init(&bars->rfree, 1);
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
      if (SAVE) ptx::tma_prefetch_desc(&tmZ);
      const uint64_t pol_x = ptx::policy_evict_first();
      const uint32_t xbytes = (uint32_t)bm * 128u;
      uint32_t unit_n = 0;
      for (int64_t u = blockIdx.x; u < nunits; u += gridDim.x, ++unit_n) {
        // the previous unit's middle tile must be dead (its last L-stage round drained)
        if (unit_n > 0 && !wait_or_abort(&bars->tmem_free, (unit_n - 1) & 1, abort_flag, status)) break;
        const int row0 = (int)(u * bm);
        for (int b = 0; b < C::NXB; ++b) {
          ptx::mbar_arrive_expect_tx(&bars->xfull[b], xbytes);
          ptx::tma_load_2d(zbuf + b * C::ATOM, &tmX, &bars->xfull[b], b * 64, row0, pol_x);
        }
        // pull the next unit's X tile into L2 while this unit computes
        if (u + gridDim.x < nunits)
          for (int b = 0; b < C::NXB; ++b) ptx::tma_prefetch_l2_2d(&tmX, b * 64, (int)((u + gridDim.x) * bm));
      }
      // no TMA load may still target this CTA's shared memory at exit
      if (unit_n > 0)
        for (int b = 0; b < C::NXB; ++b)
          ptx::mbar_wait_bounded(&bars->xfull[b], (unit_n - 1) & 1, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer (whole warp)
    constexpr uint32_t idesc1 = make_idesc(C::BM, C::OUT1);
    constexpr uint32_t idesc2 = make_idesc(C::BM, 8);
    const uint64_t z_a = make_sdesc(ptx::smem_u32(zbuf), 1024, 2);
    const uint64_t r_b = make_sdesc(ptx::smem_u32(stg), 256, 6);
    const uint64_t ring_b = make_sdesc(ptx::smem_u32(ring), 256, 6);
    uint32_t g2 = 0, unit_n = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++unit_n) {
      // TMEM is shared by both stages: the previous unit's L-stage rounds must be drained
      if (unit_n > 0 && !warp_wait_or_abort(lane, &bars->tmem_free, (unit_n - 1) & 1, abort_flag, status)) { ok = false; break; }
      ptx::tc_fence_after();
      // ---- R stage: X box b holds columns [64 b, 64 b + 64) = R slices 4 b .. 4 b + 3
      for (int b = 0; b < C::NXB; ++b) {
        if (!warp_wait_or_abort(lane, &bars->xfull[b], unit_n & 1, abort_flag, status)) { ok = false; break; }
        ptx::fence_proxy_async_smem();  // R slices were written by cp.async (generic proxy)
        ptx::tc_fence_after();
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int c = b * 64 + 16 * t;
          const int kk = c / C::IN1, s16 = (c % C::IN1) / 16;
          const uint32_t d = tmem + ((uint32_t)(kk >> 3) << 20) + (uint32_t)((kk & 7) * C::OUT1);
          ptx::mma_bf16_ss_elect(d, z_a + (uint64_t)((b * C::ATOM + 32 * t) >> 4),
                                 r_b + (uint64_t)(((4 * b + t) * C::RPIECE) >> 4), idesc1,
                                 s16 > 0 ? 1u : 0u);
        }
      }
      if (!ok) break;
      ptx::mma_commit_elect(&bars->a1_full);
      if (!warp_wait_or_abort(lane, &bars->z_full, unit_n & 1, abort_flag, status)) { ok = false; break; }
      ptx::tc_fence_after();
      // ---- L stage
      for (int r2 = 0; r2 < C::NR2 && ok; ++r2, ++g2) {
        const int slot = g2 & 1;
        if (!warp_wait_or_abort(lane, &bars->a2_empty[slot], ((g2 >> 1) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
        if (!warp_wait_or_abort(lane, &bars->lfull[slot], (g2 >> 1) & 1, abort_flag, status)) { ok = false; break; }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_after();
        const uint32_t dslot = tmem + (uint32_t)(slot * C::SLOT2);
        const uint64_t lb = ring_b + (uint64_t)((slot * C::LSTAGE) >> 4);
#pragma unroll 4
        for (int piece = 0; piece < C::LPR; ++piece) {  // piece = j * KS2 + s
          const int j = piece / C::KS2, s16 = piece % C::KS2;
          const int h = j / C::JH, jj = j % C::JH;
          const int zc = j * C::IN2 + 16 * s16;
          const uint32_t d = dslot + ((uint32_t)h << 20) + (uint32_t)(jj * 8);
          ptx::mma_bf16_ss_elect(d, z_a + (uint64_t)(((zc >> 6) * C::ATOM + (zc & 63) * 2) >> 4),
                                 lb + (uint64_t)((piece * C::LPIECE) >> 4), idesc2,
                                 s16 > 0 ? 1u : 0u);
        }
        ptx::mma_commit_elect(&bars->lempty[slot]);
        ptx::mma_commit_elect(&bars->a2_full[slot]);
      }
    }
    ptx::mma_commit_elect(&bars->mma_done);
    if (lane == 0) wait_mma_done(&bars->mma_done, abort_flag, status);
    __syncwarp();
  } else if (warp >= 2 + kWideDrainWarps) {
    // ================================================================ factor loaders
    // R slice pi = (k, s) (k = pi / (in1/16)) lands at stg + pi * RPIECE: row n of R[k] at
    // n * 32, its two 16-byte chunks swapped when (n >> 2) is odd (32B swizzle).
    // L round r2: slice j lands at stage + j * LPIECE, rows o = 8 r2 .. 8 r2 + 7.
    const int lt = (warp - 2 - kWideDrainWarps) * 32 + lane;
    const uint32_t stg_s = ptx::smem_u32(stg), ring_s = ptx::smem_u32(ring);
    uint32_t g2 = 0, unit_n = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++unit_n) {
      // R is parked in the staging buffers: the previous unit's stores must have read them
      if (unit_n > 0 && !wait_or_abort(&bars->rfree, (unit_n - 1) & 1, abort_flag, status)) { ok = false; break; }
      for (int b = 0; b < C::NXB; ++b) {
        for (int g = lt; g < 4 * C::OUT1 * 2; g += kWideLoaderThreads) {
          const int t = g / (C::OUT1 * 2), n = (g >> 1) % C::OUT1, c = g & 1;
          const int pi = 4 * b + t;
          const int col = pi * 16, k = col / C::IN1, s16 = col % C::IN1;
          ptx::cp_async_16(stg_s + pi * C::RPIECE + n * 32 + ((c ^ ((n >> 2) & 1)) << 4),
                           R + ((int64_t)k * C::OUT1 + n) * C::IN1 + s16 + c * 8);
        }
        ptx::cp_async_mbar_arrive_noinc(&bars->xfull[b]);
      }
      for (int r2 = 0; r2 < C::NR2; ++r2, ++g2) {
        const int slot = g2 & 1;
        if (!wait_or_abort(&bars->lempty[slot], ((g2 >> 1) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
        const uint32_t sb = ring_s + slot * C::LSTAGE;
        for (int g = lt; g < C::LPR * 16; g += kWideLoaderThreads) {  // 8 rows x 2 chunks per slice
          const int piece = g / 16, n = (g >> 1) & 7, c = g & 1;
          const int j = piece / C::KS2, s16 = (piece % C::KS2) * 16;
          ptx::cp_async_16(sb + piece * C::LPIECE + n * 32 + ((c ^ ((n >> 2) & 1)) << 4),
                           L + ((int64_t)j * C::OUT2 + r2 * 8 + n) * C::IN2 + s16 + c * 8);
        }
        ptx::cp_async_mbar_arrive_noinc(&bars->lfull[slot]);
      }
    }
    // no copy may still target this CTA's shared memory at exit: the copies were never
    // committed to a group (the mbarrier tracks them), so commit and wait for all of them
    ptx::cp_async_wait_all();
  } else {
    // ================================================================ drain (8 warps)
    const int quad = warp & 3, ph = (warp - 2) >> 2, half = lane >> 4;
    const int r = quad * 16 + (lane & 15);
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t z_s = ptx::smem_u32(zbuf), stg_s = ptx::smem_u32(stg);
    const bool leader = (warp == 2 && lane == 0);
    uint32_t g2 = 0, unit_n = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++unit_n) {
      // ---- R stage -> Z (over the consumed X tile)
      if (!wait_or_abort(&bars->a1_full, unit_n & 1, abort_flag, status)) { ok = false; break; }
      __syncwarp();  // the leader lane may still be coming out of the previous unit's store branch
      ptx::tc_fence_after();
#pragma unroll 1
      for (int pc = ph * C::P_HALF; pc < (ph + 1) * C::P_HALF; pc += 8) {
        float v[8][8];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          uint32_t rr[8];
          ptx::tmem_ld8(tmem + lane_off + kk * C::OUT1 + pc, rr);
#pragma unroll
          for (int e = 0; e < 8; ++e) v[kk][e] = __uint_as_float(rr[e]);
        }
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int t0 = (pc + e) * C::NB1 + half * 8;  // flat column p*nb1 + k, k = 8 half ..
          ptx::st_shared_v4(z_s + wide_chunk_off(r, t0), ptx::pack_bf16x2(v[0][e], v[1][e]),
                            ptx::pack_bf16x2(v[2][e], v[3][e]), ptx::pack_bf16x2(v[4][e], v[5][e]),
                            ptx::pack_bf16x2(v[6][e], v[7][e]));
        }
      }
      ptx::tc_fence_before();
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->z_full);
      const int row0 = (int)(u * bm);
      if (SAVE && leader) {
        // every drain warp has written and fenced its part of Z: store the tile (rows >= bm
        // of a tile are not part of the box)
        if (!wait_or_abort(&bars->z_full, unit_n & 1, abort_flag, status)) {
          ok = false;
        } else {
          for (int a = 0; a < C::ZATOMS; ++a) ptx::tma_store_2d(&tmZ, zbuf + a * C::ATOM, a * 64, row0);
          ptx::bulk_commit_group();
        }
      }
      // ---- L-stage rounds -> staged output runs
      for (int r2 = 0; r2 < C::NR2 && ok; ++r2, ++g2) {
        const int slot = g2 & 1;
        if (!wait_or_abort(&bars->a2_full[slot], (g2 >> 1) & 1, abort_flag, status)) { ok = false; break; }
        // staging buffer `slot` was last used two rounds ago; its stores must have read it
        if (leader) {
          ptx::bulk_wait_read_allbut1();
          ptx::mbar_arrive(&bars->stg_free);
        }
        if (!wait_or_abort(&bars->stg_free, g2 & 1, abort_flag, status)) { ok = false; break; }
        __syncwarp();  // tcgen05.ld is warp-collective
        ptx::tc_fence_after();
        const uint32_t tb = tmem + lane_off + (uint32_t)(slot * C::SLOT2);
        const uint32_t sb = stg_s + (uint32_t)(slot * C::STG_BYTES);
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
            ptx::st_shared_v4(sb + wide_chunk_off(r, lc), ptx::pack_bf16x2(v[0][e], v[1][e]),
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
          if (!wait_or_abort(&bars->staged, g2 & 1, abort_flag, status)) {
            ok = false;
          } else {
            for (int a = 0; a < C::OATOMS; ++a)
              ptx::tma_store_2d(&tmY, stg + slot * C::STG_BYTES + a * C::ATOM, r2 * C::OW + a * 64, row0);
            ptx::bulk_commit_group();
          }
        }
      }
      if (!ok) break;
      // with SAVE, the next unit's X may overwrite Z only once the Z stores (the group before
      // the last round's) have read it
      if (SAVE && leader) ptx::bulk_wait_read_allbut1();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->tmem_free);
      if (leader) {
        // the staging buffers take the next unit's R once these stores have read them
        ptx::bulk_wait_read_all();
        ptx::mbar_arrive(&bars->rfree);
      }
    }
    if (leader) ptx::bulk_wait_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

// Rows per unit: a multiple of 8, at most 64, chosen so the units fill the SMs in as few
// equal waves as possible (e.g. 8192 rows on 148 SMs: 56-row tiles, 147 units).
static int balanced_bm(int64_t rows, int nsm) {
  const int64_t per_wave = (int64_t)64 * nsm;
  const int64_t waves = (rows + per_wave - 1) / per_wave;
  const int64_t per_unit = (rows + waves * nsm - 1) / (waves * nsm);
  int64_t bm = (per_unit + 7) / 8 * 8;
  if (bm > 64) bm = 64;
  if (bm < 8) bm = 8;
  return (int)bm;
}

template <class C, int SAVE>
static cudaError_t launch_wide(const void* X, const void* R, const void* L, void* Y, void* Z, int64_t rows,
                               int* status, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const int nsm = num_sms();
  const int bm = balanced_bm(rows, nsm);
  CUtensorMap mX, mY, mZ;
  if (!make_map_2d(&mX, X, C::N_IN, (uint64_t)rows, 64, (uint32_t)bm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mY, Y, C::N_OUT, (uint64_t)rows, 64, (uint32_t)bm, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (SAVE && !make_map_2d(&mZ, Z, C::N_MID, (uint64_t)rows, 64, (uint32_t)bm, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!SAVE) mZ = mY;  // unused
  cudaError_t e = ensure_smem_attr((const void*)tc_wide_kernel<C, SAVE>, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int64_t nunits = (rows + bm - 1) / bm;
  const int64_t grid = nunits < nsm ? nunits : nsm;
  return launch_kernel(tc_wide_kernel<C, SAVE>, dim3((unsigned)grid), dim3(kWideThreads), C::SMEM_BYTES, st,
                       false, mX, mY, mZ, (const __nv_bfloat16*)R, (const __nv_bfloat16*)L, rows, bm, status);
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
  if (wide_shape_is<WideR768>(s)) return launch_wide<WideR768, 0>(X, R, L, Y, nullptr, s.rows, status, st);
  return cudaErrorNotSupported;
}

cudaError_t tc_wide_fwd_save(const void* X, const void* R, const void* L, void* Y, void* Z, const Shape& s,
                             int* status, cudaStream_t st) {
  if (wide_shape_is<WideR768>(s)) return launch_wide<WideR768, 1>(X, R, L, Y, Z, s.rows, status, st);
  return cudaErrorNotSupported;
}

}  // namespace monarch
