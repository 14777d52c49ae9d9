// Fused Monarch forward for small blocks (out1, out2 <= 32): one row tile of X (at most 64 rows)
// per unit and the whole middle vector on chip, on the tcgen05 tensor cores.
//
// Per unit (bm <= 64 rows; the MMAs always cover 64, rows >= bm of a tile are never stored):
//   1. R stage: X tile (TMA, 128B swizzle, 64-column boxes) x R[k]^T, M = 64 MMAs.
//      A round covers 16 blocks k: blocks k0..k0+7 accumulate at TMEM lane offset 0
//      and k0+8..k0+15 at lane offset 16 (the two halves of the M = 64 data-path
//      layout), so each drain thread owns 8 consecutive k of one row.
//   2. Permutation P on chip: the drain threads round u[k][p] to bf16 and store the
//      8 consecutive k as one 16-byte chunk at flat column p*nb1 + k of the Z tile
//      (shared memory, 128B-swizzled K-major: the layout the next MMA reads).
//   3. L stage: Z_j x L[j]^T, M = 64 MMAs, same lane-offset pairing over j.
//   4. Output permutation: the drain threads write v[j][o] as 16-byte chunks (8
//      consecutive j, or 8 consecutive o when there is no output transpose) into a
//      full-row output tile staged in the (now dead) Z buffer; one thread then
//      writes it with TMA tensor stores of whole 128-byte row segments.
// X is read once, Y is written as full rows, and the intermediate never leaves the
// SM.  Roles: warp 0 TMA producer (X boxes), warp 1 MMA issuer and TMEM owner,
// warps 2..9 drain (two warps per TMEM lane quadrant, splitting the columns of a
// round), warps 10..13 weight loaders.  The weight slices are copied with
// 16-byte cp.async (LSU path, coalesced global reads, software 32B swizzle on the
// shared-memory side) so that the TMA engine only moves 128-byte rows of X and Y:
// TMA throughput is set by rows per cycle, and weight slices have 32-byte rows.
// All waits are bounded (see tc_common.cuh).
#include "tc_common.cuh"

namespace monarch {

constexpr int kRowsThreads = 448;  // 14 warps
constexpr int kRowsDrainWarps = 8;
constexpr int kRowsLoaderWarps = 4;
constexpr int kRowsLoaderThreads = kRowsLoaderWarps * 32;

// MODE 0: Y only.  MODE 1: Y, and the middle tile (bf16, block-contiguous) is also
// stored through tmZ.  MODE 2: R stage and permutation only; the middle tile is the
// output (tmZ).
template <int NB1_, int IN1_, int OUT1_, int NB2_, int IN2_, int OUT2_, int OT_, int MODE_ = 0>
struct RowsCfg {
  static constexpr int NB1 = NB1_, IN1 = IN1_, OUT1 = OUT1_;
  static constexpr int NB2 = NB2_, IN2 = IN2_, OUT2 = OUT2_, OT = OT_, MODE = MODE_;
  static constexpr int N_IN = NB1 * IN1, N_MID = NB1 * OUT1, N_OUT = NB2 * OUT2;
  static constexpr int BM = 64;
  static constexpr int KS1 = IN1 / 16, KS2 = IN2 / 16;
  static constexpr int NR1 = NB1 / 16, NR2 = NB2 / 16;  // rounds of 16 blocks
  static constexpr int SLOT1 = 8 * OUT1, SLOT2 = 8 * OUT2;
  static constexpr int SLOT = SLOT1 > SLOT2 ? SLOT1 : SLOT2;  // TMEM columns per slot
  static constexpr int TMEM_COLS = 2 * SLOT <= 32 ? 32 : (2 * SLOT <= 64 ? 64 : (2 * SLOT <= 128 ? 128 : (2 * SLOT <= 256 ? 256 : 512)));
  static constexpr int NXB = N_IN / 64;
  static constexpr int XBOX_BYTES = BM * 128;  // 64 rows x 64 columns
  static constexpr int RPIECE = OUT1 * 32;     // R[k] rows x one 16-wide K slice, 32B swizzle
  static constexpr int LPIECE = OUT2 * 32;
  static constexpr int STAGE_BYTES = XBOX_BYTES + 4 * RPIECE;
  static constexpr int PPR = 16 * KS2;  // L slices per L-stage round
  static constexpr int LPS_MAX = STAGE_BYTES / LPIECE;
  // L slices per ring stage: the largest divisor of PPR that fits, so stages never straddle rounds
  static constexpr int LPS = LPS_MAX >= PPR ? PPR : (LPS_MAX >= PPR / 2 ? PPR / 2 : (LPS_MAX >= PPR / 4 ? PPR / 4 : (LPS_MAX >= PPR / 8 ? PPR / 8 : PPR / 16)));
  static constexpr int SPR = PPR / LPS;   // ring stages per L-stage round
  static constexpr int NPIECE2 = NB2 * KS2;
  static constexpr int NSTAGE2 = MODE == 2 ? 0 : NR2 * SPR;
  static constexpr int BPR = IN1 / 4;     // X boxes (64 columns) per R-stage round of 16 blocks
  static constexpr int ATOM_BYTES = BM * 128;  // 64 rows x 64 bf16 columns
  static constexpr int ZATOMS = N_MID / 64;
  static constexpr int OATOMS = N_OUT / 64;
  static constexpr int Z_BYTES = ZATOMS * ATOM_BYTES;
  static constexpr int BAR_BYTES = 1024;
  static constexpr int NSTAGE_RAW = (kSmemBudget - Z_BYTES - BAR_BYTES) / STAGE_BYTES;
  static constexpr int NSTAGE = NSTAGE_RAW > 12 ? 12 : NSTAGE_RAW;
  static constexpr int SMEM_BYTES = Z_BYTES + NSTAGE * STAGE_BYTES + BAR_BYTES + 1024;
  static constexpr int P_HALF = OUT1 / 2, O_HALF = OUT2 / 2;

  static_assert(NB1 % 16 == 0 && NB2 % 16 == 0, "rounds of 16 blocks");
  static_assert(OUT1 % 16 == 0 && OUT2 % 16 == 0 && OUT1 <= 32 && OUT2 <= 32, "small blocks");
  static_assert(IN1 % 16 == 0 && IN2 % 16 == 0, "K steps of 16");
  static_assert(N_IN % 64 == 0 && N_MID % 64 == 0 && N_OUT % 64 == 0, "64-column atoms");
  static_assert(OATOMS <= ZATOMS, "output tile is staged in the Z buffer");
  static_assert(NR2 <= 2, "all L-stage rounds must fit the two TMEM slots");
  static_assert(NSTAGE >= 3, "shared memory");
  static_assert(LPS >= 1 && PPR % LPS == 0, "L slices per stage");
  static_assert(NXB == NR1 * BPR, "R-stage rounds align with X boxes");
};

struct RowsBars {
  uint64_t full[12], empty[12];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t z_full, zfree, staged, zsaved, mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

// Byte offset of the 16-byte chunk holding columns [c, c+8) of row r in a tile of
// 64-column, 128B-swizzled atoms (64 rows x 128 bytes each).
__device__ __forceinline__ uint32_t atom_chunk_off(int r, int c) {
  const uint32_t chunk = (uint32_t)((c & 63) >> 3);
  return (uint32_t)(c >> 6) * (64 * 128) + (uint32_t)(r >> 3) * 1024 + (uint32_t)(r & 7) * 128 +
         ((chunk ^ (uint32_t)(r & 7)) << 4);
}

template <class C>
__global__ void __launch_bounds__(kRowsThreads, 1)
    tc_rows_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                   const __grid_constant__ CUtensorMap tmZ,
                   const __nv_bfloat16* __restrict__ R, const __nv_bfloat16* __restrict__ L,
                   int64_t rows, int bm, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* zbuf = smem;  // Z tile, later the output staging tile
  uint8_t* ring = smem + C::Z_BYTES;
  RowsBars* bars = (RowsBars*)(ring + C::NSTAGE * C::STAGE_BYTES);
  int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t nunits = (rows + bm - 1) / bm;  // units of bm <= 64 rows (MMAs always cover 64)

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      // producer arrive (+ X bytes) and one cp.async completion arrival per loader thread
      ptx::mbar_init(&bars->full[i], 1 + kRowsLoaderThreads);
      ptx::mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->acc_full[i], 1);
      ptx::mbar_init(&bars->acc_empty[i], kRowsDrainWarps);
    }
    ptx::mbar_init(&bars->z_full, kRowsDrainWarps);
    ptx::mbar_init(&bars->zfree, kRowsDrainWarps);
    ptx::mbar_init(&bars->staged, kRowsDrainWarps);
    ptx::mbar_init(&bars->zsaved, 1);
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
  // launched with programmatic stream serialization inside the backward: the inputs are
  // written by the previous kernels of the stream
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  if (warp == 0) {
    // ================================================================ TMA producer (X)
    if (lane == 0) {
      ptx::tma_prefetch_desc(&tmX);
      if (C::MODE != 2) ptx::tma_prefetch_desc(&tmY);
      if (C::MODE != 0) ptx::tma_prefetch_desc(&tmZ);
      const uint64_t pol_x = ptx::policy_evict_first();
      uint32_t it = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
        const int row0 = (int)(u * bm);
        for (int b = 0; b < C::NXB; ++b, ++it) {
          const int st = it % C::NSTAGE;
          if (!wait_or_abort(&bars->empty[st], ((it / C::NSTAGE) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(&bars->full[st], (uint32_t)bm * 128u);  // a box of bm rows
          ptx::tma_load_2d(ring + st * C::STAGE_BYTES, &tmX, &bars->full[st], b * 64, row0, pol_x);
        }
        // this unit's X is on its way: pull the next unit's X tile into L2 now, so that HBM
        // streams it during this unit's L stage and stores instead of after them
        if (ok && u + gridDim.x < nunits)
          for (int b = 0; b < C::NXB; ++b) ptx::tma_prefetch_l2_2d(&tmX, b * 64, (int)((u + gridDim.x) * bm));
        for (int sp = 0; sp < C::NSTAGE2 && ok; ++sp, ++it) {
          const int st = it % C::NSTAGE;
          if (!wait_or_abort(&bars->empty[st], ((it / C::NSTAGE) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
          ptx::mbar_arrive(&bars->full[st]);  // L stages carry no TMA bytes
        }
      }
      const uint32_t issued = it;
      for (uint32_t k = (issued > (uint32_t)C::NSTAGE ? issued - C::NSTAGE : 0); k < issued; ++k)
        ptx::mbar_wait_bounded(&bars->full[k % C::NSTAGE], (k / C::NSTAGE) & 1, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // The whole warp runs this loop (warp-uniform scalar work); elect.sync picks the
    // issuing lane.  Descriptors are precomputed bases plus constant offsets.
    constexpr uint32_t idesc1 = make_idesc(C::BM, C::OUT1);
    constexpr uint32_t idesc2 = make_idesc(C::BM, C::OUT2);
    const uint64_t ring_a = make_sdesc(ptx::smem_u32(ring), 1024, 2);  // X boxes, 128B swizzle
    const uint64_t ring_b = make_sdesc(ptx::smem_u32(ring), 256, 6);   // weight slices, 32B swizzle
    const uint64_t z_a = make_sdesc(ptx::smem_u32(zbuf), 1024, 2);     // Z tile, 128B swizzle
    uint32_t it = 0, rnd = 0, unit_n = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++unit_n) {
      // ---- R stage: round r1 covers blocks [16 r1, 16 r1 + 16) = BPR X boxes
      for (int r1 = 0; r1 < C::NR1 && ok; ++r1, ++rnd) {
        const int slot = rnd & 1;
        if (!warp_wait_or_abort(lane, &bars->acc_empty[slot], ((rnd >> 1) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t dslot = tmem + slot * C::SLOT;
        for (int bb = 0; bb < C::BPR; ++bb, ++it) {
          const int st = it % C::NSTAGE;
          if (!warp_wait_or_abort(lane, &bars->full[st], (it / C::NSTAGE) & 1, abort_flag, status)) { ok = false; break; }
          ptx::fence_proxy_async_smem();  // weight slices were written by cp.async (generic proxy)
          ptx::tc_fence_after();
          const uint64_t soff = (uint64_t)((st * C::STAGE_BYTES) >> 4);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int c = bb * 64 + 16 * t;  // column within the round
            const int kk = c / C::IN1, s16 = (c % C::IN1) / 16;
            const uint32_t d = dslot + ((uint32_t)(kk >> 3) << 20) + (uint32_t)((kk & 7) * C::OUT1);
            ptx::mma_bf16_ss_elect(d, ring_a + soff + (uint64_t)((32 * t) >> 4),
                                   ring_b + soff + (uint64_t)((C::XBOX_BYTES + t * C::RPIECE) >> 4),
                                   idesc1, s16 > 0 ? 1u : 0u);
          }
          ptx::mma_commit_elect(&bars->empty[st]);  // the box is free once these MMAs finish
        }
        if (!ok) break;
        ptx::mma_commit_elect(&bars->acc_full[slot]);
      }
      if (!ok) break;
      if (C::MODE == 2) continue;  // no L stage
      if (!warp_wait_or_abort(lane, &bars->z_full, unit_n & 1, abort_flag, status)) { ok = false; break; }
      ptx::tc_fence_after();
      // ---- L stage: round r2 covers blocks [16 r2, 16 r2 + 16), SPR ring stages of LPS slices
      for (int r2 = 0; r2 < C::NR2 && ok; ++r2, ++rnd) {
        const int slot = rnd & 1;
        if (!warp_wait_or_abort(lane, &bars->acc_empty[slot], ((rnd >> 1) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t dslot = tmem + slot * C::SLOT;
        for (int sp = 0; sp < C::SPR; ++sp, ++it) {
          const int st = it % C::NSTAGE;
          if (!warp_wait_or_abort(lane, &bars->full[st], (it / C::NSTAGE) & 1, abort_flag, status)) { ok = false; break; }
          ptx::fence_proxy_async_smem();  // weight slices were written by cp.async (generic proxy)
          ptx::tc_fence_after();
          const uint64_t soff = (uint64_t)((st * C::STAGE_BYTES) >> 4);
#pragma unroll
          for (int t = 0; t < C::LPS; ++t) {
            const int piece = sp * C::LPS + t;  // within the round: jj * KS2 + s
            const int jj = piece / C::KS2, s16 = piece % C::KS2;
            const int zc = (r2 * 16 + jj) * C::IN2 + 16 * s16;
            const uint32_t d = dslot + ((uint32_t)(jj >> 3) << 20) + (uint32_t)((jj & 7) * C::OUT2);
            ptx::mma_bf16_ss_elect(d, z_a + (uint64_t)(((zc >> 6) * C::ATOM_BYTES + (zc & 63) * 2) >> 4),
                                   ring_b + soff + (uint64_t)((t * C::LPIECE) >> 4), idesc2,
                                   s16 > 0 ? 1u : 0u);
          }
          ptx::mma_commit_elect(&bars->empty[st]);
        }
        if (!ok) break;
        ptx::mma_commit_elect(&bars->acc_full[slot]);
      }
    }
    ptx::mma_commit_elect(&bars->mma_done);
    if (lane == 0) wait_mma_done(&bars->mma_done, abort_flag, status);
    __syncwarp();
  } else if (warp >= 2 + kRowsDrainWarps) {
    // ================================================================ weight loaders
    // Each stage gets its weight slices (R slices of the X box's four K steps, or
    // LPS slices of L) as 16-byte cp.async chunks written in the 32B-swizzled
    // K-major layout: chunk c of row n of a slice lands at n*32 + ((c ^ ((n>>2)&1)) << 4).
    // Every loader thread then arrives on the stage's full barrier when its own
    // copies have landed (cp.async.mbarrier.arrive.noinc); the MMA warp fences the
    // async proxy after observing the barrier.
    const int lt = (warp - 2 - kRowsDrainWarps) * 32 + lane;
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
          for (int g = lt; g < 4 * C::OUT1 * 2; g += kRowsLoaderThreads) {
            const int t = g / (C::OUT1 * 2), n = (g >> 1) % C::OUT1, c = g & 1;
            const int col = b * 64 + t * 16;
            const int k = col / C::IN1, s16 = col % C::IN1;
            ptx::cp_async_16(sb + C::XBOX_BYTES + t * C::RPIECE + n * 32 + ((c ^ ((n >> 2) & 1)) << 4),
                             R + ((int64_t)k * C::OUT1 + n) * C::IN1 + s16 + c * 8);
          }
        } else {
          const int p0 = (sq - C::NXB) * C::LPS;
          const int np = (C::NPIECE2 - p0) < C::LPS ? (C::NPIECE2 - p0) : C::LPS;
          for (int g = lt; g < np * C::OUT2 * 2; g += kRowsLoaderThreads) {
            const int t = g / (C::OUT2 * 2), n = (g >> 1) % C::OUT2, c = g & 1;
            const int pi = p0 + t, j = pi / C::KS2, s16 = (pi % C::KS2) * 16;
            ptx::cp_async_16(sb + t * C::LPIECE + n * 32 + ((c ^ ((n >> 2) & 1)) << 4),
                             L + ((int64_t)j * C::OUT2 + n) * C::IN2 + s16 + c * 8);
          }
        }
        ptx::cp_async_mbar_arrive_noinc(&bars->full[st]);
      }
    }
    ptx::cp_async_wait_all();  // no copy may still target this CTA's shared memory at exit
  } else {
    // ================================================================ drain (8 warps)
    const int quad = warp & 3;              // TMEM lane quadrant of this warp
    const int ph = (warp - 2) >> 2;         // which half of a round's columns
    const int half = lane >> 4;             // lane offset 0 / 16 -> block half
    const int r = quad * 16 + (lane & 15);  // row within the 64-row tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t z_s = ptx::smem_u32(zbuf);
    const bool leader = (warp == 2 && lane == 0);
    uint32_t rnd = 0, unit_n = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++unit_n) {
      // ---- R-stage rounds -> Z
      for (int r1 = 0; r1 < C::NR1 && ok; ++r1, ++rnd) {
        const int slot = rnd & 1;
        if (!wait_or_abort(&bars->acc_full[slot], (rnd >> 1) & 1, abort_flag, status)) { ok = false; break; }
        if (r1 == 0) {
          // the previous unit's output stores must have finished reading the Z buffer
          if (leader) ptx::bulk_wait_read_all();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&bars->zfree);
          if (!wait_or_abort(&bars->zfree, unit_n & 1, abort_flag, status)) { ok = false; break; }
        }
        ptx::tc_fence_after();
        const uint32_t tb = tmem + lane_off + slot * C::SLOT;
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
            const int t0 = (pc + e) * C::NB1 + r1 * 16 + half * 8;  // flat column of k = r1*16 + 8*half
            ptx::st_shared_v4(z_s + atom_chunk_off(r, t0), ptx::pack_bf16x2(v[0][e], v[1][e]),
                              ptx::pack_bf16x2(v[2][e], v[3][e]), ptx::pack_bf16x2(v[4][e], v[5][e]),
                              ptx::pack_bf16x2(v[6][e], v[7][e]));
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->acc_empty[slot]);
      }
      if (!ok) break;
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (C::MODE == 2) {
        // the middle tile is the output: hand it to the TMA store engine
        if (lane == 0) ptx::mbar_arrive(&bars->staged);
        if (leader) {
          if (!wait_or_abort(&bars->staged, unit_n & 1, abort_flag, status)) {
            ok = false;
          } else {
            const int row0 = (int)(u * bm);
            for (int a = 0; a < C::ZATOMS; ++a) ptx::tma_store_2d(&tmZ, zbuf + a * C::ATOM_BYTES, a * 64, row0);
            ptx::bulk_commit_group();
          }
        }
        continue;
      }
      if (lane == 0) ptx::mbar_arrive(&bars->z_full);
      if (C::MODE == 1) {
        // side output of the middle tile; it must be read out before the staging reuses it
        if (lane == 0) ptx::mbar_arrive(&bars->staged);
        if (leader) {
          // `staged` completes twice per unit in this mode: phase 2n (middle tile), 2n+1 (Y)
          if (wait_or_abort(&bars->staged, 0u, abort_flag, status)) {
            const int row0 = (int)(u * bm);
            for (int a = 0; a < C::ZATOMS; ++a) ptx::tma_store_2d(&tmZ, zbuf + a * C::ATOM_BYTES, a * 64, row0);
            ptx::bulk_commit_group();
            ptx::bulk_wait_read_all();
          }
          ptx::mbar_arrive(&bars->zsaved);
        }
      }
      // ---- L-stage rounds: wait for all of them (Z is then dead), stage the output rows
      const uint32_t rnd0 = rnd;
      for (int r2 = 0; r2 < C::NR2 && ok; ++r2)
        if (!wait_or_abort(&bars->acc_full[(rnd0 + r2) & 1], ((rnd0 + r2) >> 1) & 1, abort_flag, status)) ok = false;
      if (!ok) break;
      if (C::MODE == 1 && !wait_or_abort(&bars->zsaved, unit_n & 1, abort_flag, status)) { ok = false; break; }
      ptx::tc_fence_after();
      for (int r2 = 0; r2 < C::NR2; ++r2, ++rnd) {
        const uint32_t tb = tmem + lane_off + (rnd & 1) * C::SLOT;
#pragma unroll 1
        for (int oc = ph * C::O_HALF; oc < (ph + 1) * C::O_HALF; oc += 8) {
          float v[8][8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            uint32_t rr[8];
            ptx::tmem_ld8(tb + jj * C::OUT2 + oc, rr);
#pragma unroll
            for (int e = 0; e < 8; ++e) v[jj][e] = __uint_as_float(rr[e]);
          }
          ptx::tmem_wait_ld();
          const int jb = r2 * 16 + half * 8;
          if (C::OT == 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {  // y[o*nb2 + j], 8 consecutive j
              const int c = (oc + e) * C::NB2 + jb;
              ptx::st_shared_v4(z_s + atom_chunk_off(r, c), ptx::pack_bf16x2(v[0][e], v[1][e]),
                                ptx::pack_bf16x2(v[2][e], v[3][e]), ptx::pack_bf16x2(v[4][e], v[5][e]),
                                ptx::pack_bf16x2(v[6][e], v[7][e]));
            }
          } else {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {  // y[j*out2 + o], 8 consecutive o
              const int c = (jb + jj) * C::OUT2 + oc;
              ptx::st_shared_v4(z_s + atom_chunk_off(r, c), ptx::pack_bf16x2(v[jj][0], v[jj][1]),
                                ptx::pack_bf16x2(v[jj][2], v[jj][3]), ptx::pack_bf16x2(v[jj][4], v[jj][5]),
                                ptx::pack_bf16x2(v[jj][6], v[jj][7]));
            }
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->acc_empty[rnd & 1]);
      }
      // ---- hand the staged rows to the TMA store engine
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->staged);
      if (leader) {
        if (!wait_or_abort(&bars->staged, C::MODE == 1 ? 1u : (unit_n & 1), abort_flag, status)) {
          ok = false;
        } else {
          const int row0 = (int)(u * bm);
          for (int a = 0; a < C::OATOMS; ++a) ptx::tma_store_2d(&tmY, zbuf + a * C::ATOM_BYTES, a * 64, row0);
          ptx::bulk_commit_group();
        }
      }
    }
    if (leader) ptx::bulk_wait_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

// Run one row-tile kernel.  X: (rows, N_IN) input; W1 (nb1, out1, in1) and W2
// (nb2, out2, in2) the stage weights in the forward layout; Y (rows, N_OUT) output
// (MODE 0/1); Zout (rows, N_MID) middle tile (MODE 1/2).
// Rows per unit: a multiple of 8, at most 64, chosen so the units fill the SMs in as few equal
// waves as possible (16384 rows on 148 SMs: 56-row units, two a CTA, against 64-row units of which
// 40 CTAs get one and 108 get two).  A unit's time is its dependency chain, so the slowest CTA
// sets the kernel's.
static int rows_unit_bm(int64_t rows, int nsm) {
  const int64_t per_wave = (int64_t)64 * nsm;
  const int64_t waves = (rows + per_wave - 1) / per_wave;
  const int64_t per_unit = (rows + waves * nsm - 1) / (waves * nsm);
  int64_t bm = (per_unit + 7) / 8 * 8;
  if (bm > 64) bm = 64;
  if (bm < 8) bm = 8;
  return (int)bm;
}

template <class C>
static cudaError_t launch_rows(const void* X, const void* W1, const void* W2, void* Y, void* Zout,
                               int64_t rows, int* status, cudaStream_t st, bool pdl = false) {
  if (rows == 0) return cudaSuccess;
  const int bm = rows_unit_bm(rows, num_sms());
  CUtensorMap mX, mY, mZ;
  if (!make_map_2d(&mX, X, C::N_IN, (uint64_t)rows, 64, (uint32_t)bm, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  mY = mX;
  mZ = mX;
  if (C::MODE != 2 &&
      !make_map_2d(&mY, Y, C::N_OUT, (uint64_t)rows, 64, (uint32_t)bm, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (C::MODE != 0 &&
      !make_map_2d(&mZ, Zout, C::N_MID, (uint64_t)rows, 64, (uint32_t)bm, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_attr((const void*)tc_rows_kernel<C>, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int64_t nunits = (rows + bm - 1) / bm;
  int64_t grid = num_sms();
  if (grid > nunits) grid = nunits;
  return launch_kernel(tc_rows_kernel<C>, dim3((unsigned)grid), dim3(kRowsThreads), C::SMEM_BYTES, st,
                       pdl, mX, mY, mZ, (const __nv_bfloat16*)W1, (const __nv_bfloat16*)W2, rows, bm, status);
}

using RowsSq16 = RowsCfg<16, 16, 16, 16, 16, 16, 1>;  // n = 256 = 16^2
using RowsSq32 = RowsCfg<32, 32, 32, 32, 32, 32, 1>;  // n = 1024 = 32^2
// Backward of the square shapes (in2 == nb1, out1 == nb2): the dual map
// dU = P^-1 (L^T-stage(dV)), dX = R^T-stage(dU) is a row-tile map with the
// transposed factors and no output transpose; MODE 1 also stores dU.
using RowsSq16Bwd = RowsCfg<16, 16, 16, 16, 16, 16, 0, 1>;
using RowsSq32Bwd = RowsCfg<32, 32, 32, 32, 32, 32, 0, 1>;
// Training forward: Y, and the middle tile Z (block-contiguous by L block) stored for the backward.
using RowsSq16Save = RowsCfg<16, 16, 16, 16, 16, 16, 1, 1>;
using RowsSq32Save = RowsCfg<32, 32, 32, 32, 32, 32, 1, 1>;
// R stage and permutation only (Z = P R x), for the weight gradient of L.
using RowsSq16Z = RowsCfg<16, 16, 16, 16, 16, 16, 1, 2>;
using RowsSq32Z = RowsCfg<32, 32, 32, 32, 32, 32, 1, 2>;

template <class C>
static bool rows_shape_is(const Shape& s) {
  return s.nb1 == C::NB1 && s.in1 == C::IN1 && s.out1 == C::OUT1 && s.nb2 == C::NB2 &&
         s.in2 == C::IN2 && s.out2 == C::OUT2 && s.out_transpose == C::OT;
}

bool tc_rows_supported(const Shape& s) {
  return rows_shape_is<RowsSq16>(s) || rows_shape_is<RowsSq32>(s);
}

cudaError_t tc_rows_fwd(const void* X, const void* R, const void* L, void* Y, const Shape& s,
                        int* status, cudaStream_t st) {
  if (rows_shape_is<RowsSq16>(s)) return launch_rows<RowsSq16>(X, R, L, Y, nullptr, s.rows, status, st);
  if (rows_shape_is<RowsSq32>(s)) return launch_rows<RowsSq32>(X, R, L, Y, nullptr, s.rows, status, st);
  return cudaErrorNotSupported;
}

// Y = X M^T and, on the side, Z = P R x (what the middle-only pass of the backward computes).
cudaError_t tc_rows_fwd_save(const void* X, const void* R, const void* L, void* Y, void* Z, const Shape& s,
                             int* status, cudaStream_t st) {
  if (rows_shape_is<RowsSq16>(s)) return launch_rows<RowsSq16Save>(X, R, L, Y, Z, s.rows, status, st);
  if (rows_shape_is<RowsSq32>(s)) return launch_rows<RowsSq32Save>(X, R, L, Y, Z, s.rows, status, st);
  return cudaErrorNotSupported;
}

// Z = P R x for every row (block-contiguous middle vector, bf16).
cudaError_t tc_rows_middle(const void* X, const void* R, void* Z, const Shape& s, int* status,
                           cudaStream_t st) {
  if (rows_shape_is<RowsSq16>(s)) return launch_rows<RowsSq16Z>(X, R, nullptr, nullptr, Z, s.rows, status, st, true);
  if (rows_shape_is<RowsSq32>(s)) return launch_rows<RowsSq32Z>(X, R, nullptr, nullptr, Z, s.rows, status, st, true);
  return cudaErrorNotSupported;
}

// dX and dU from the block-contiguous dV with the transposed factors Lt, Rt.
cudaError_t tc_rows_dual(const void* dV, const void* Lt, const void* Rt, void* dX, void* dU,
                         const Shape& s, int* status, cudaStream_t st) {
  if (rows_shape_is<RowsSq16>(s)) return launch_rows<RowsSq16Bwd>(dV, Lt, Rt, dX, dU, s.rows, status, st, true);
  if (rows_shape_is<RowsSq32>(s)) return launch_rows<RowsSq32Bwd>(dV, Lt, Rt, dX, dU, s.rows, status, st, true);
  return cudaErrorNotSupported;
}

}  // namespace monarch
