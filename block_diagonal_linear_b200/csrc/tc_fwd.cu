// Fused Monarch forward on the 5th-generation tensor cores (sm_100a, tcgen05).
//
// One CTA (persistent, one per SM) processes "units": a tile of BM = 128 rows
// of X and one group of G output blocks j of L.  A group needs Z[j][q] for its
// j's, i.e. the flat middle positions t in [g*G*in2, (g+1)*G*in2), which come
// from R output rows p in [g*NP, (g+1)*NP) of EVERY R block (NP = G*in2/nb1).
// Per unit:
//   1. R stage: X tile (TMA, 128B swizzle) x R[k][p-range]^T on tcgen05 into TMEM
//      (fp32), nb1 block-GEMMs of 128 x NP x in1.
//   2. Permutation P on chip: drain warps read u[k][p] from TMEM, round to bf16
//      and store it at local flat column (p - p0)*nb1 + k of the Z tile in shared
//      memory (128B-swizzled K-major, the layout the next MMA reads).  Z never
//      goes to HBM.
//   3. L stage: Z_j (smem) x L[j]^T on tcgen05 into TMEM, G block-GEMMs of
//      128 x out2 x in2.
//   4. Output permutation: drain warps store v[j][o] at y[o*nb2 + j] (or
//      y[j*out2 + o]) with 16-byte (8 consecutive j / o) vector stores.
// Roles: warp 0 = TMA producer, warp 1 = MMA issuer (+ TMEM owner),
// warps 2..5 = TMEM drain (one thread per row).  A ring of shared-memory
// stages carries X boxes with the matching R slices (R stage) and L slices
// (L stage).  Two 256-column TMEM slots double-buffer the accumulators.
// Every mbarrier wait is bounded; on timeout the CTA records
// kStatusTimeout, skips the rest of its work, waits for its own copies and
// MMAs, frees TMEM and returns.
#include "tc_common.cuh"

namespace monarch {

constexpr int kTcThreads = 192;

struct Bars {
  uint64_t full[8], empty[8];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t z_full, z_empty, mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

template <int NB1_, int IN1_, int OUT1_, int NB2_, int IN2_, int OUT2_, int OT_, int G_>
struct FwdCfg {
  static constexpr int NB1 = NB1_, IN1 = IN1_, OUT1 = OUT1_;
  static constexpr int NB2 = NB2_, IN2 = IN2_, OUT2 = OUT2_, OT = OT_, G = G_;
  static constexpr int N_IN = NB1 * IN1, N_MID = NB1 * OUT1, N_OUT = NB2 * OUT2;
  static constexpr int NGROUPS = NB2 / G;
  static constexpr int NP = G * IN2 / NB1;  // R output rows per block used by one group
  static constexpr int ZCOLS = G * IN2;     // local middle width of one group
  static constexpr int BM = 128;
  static constexpr int SLOT = 256;          // TMEM columns per accumulator slot
  // R stage rounds: KR blocks of NP columns each per slot
  static constexpr int KR = (NB1 * NP <= SLOT) ? NB1 : SLOT / NP;
  static constexpr int NR1 = NB1 / KR;
  static constexpr int KS1 = IN1 / 16;
  // L stage: MMA N = OC, rounds of JR blocks x OC columns
  static constexpr int OC = OUT2 < 256 ? OUT2 : 256;
  static constexpr int NOC = OUT2 / OC;
  static constexpr int JR = (OUT2 <= SLOT) ? ((SLOT / OUT2) < G ? (SLOT / OUT2) : G) : 1;
  static constexpr int NR2 = (G / JR) * NOC;
  static constexpr int KS2 = IN2 / 16;
  // shared memory
  static constexpr int NXB = (N_IN + 63) / 64;  // 64-column X boxes per tile
  static constexpr int XBOX_BYTES = BM * 128;
  static constexpr int RPIECE = NP * 32;        // one 16-wide K slice of NP rows of R (32B swizzle)
  static constexpr int LPIECE = OC * 32;        // one 16-wide K slice of OC rows of L
  static constexpr int STAGE_BYTES = XBOX_BYTES + 4 * RPIECE;
  static constexpr int LPS = STAGE_BYTES / LPIECE;  // L slices per stage
  static constexpr int NPIECE2 = G * KS2 * NOC;
  static constexpr int NSTAGE2 = (NPIECE2 + LPS - 1) / LPS;  // stages of the L stage per unit
  static constexpr int ZATOMS = (ZCOLS + 63) / 64;
  static constexpr int Z_BYTES = ZATOMS * BM * 128;
  static constexpr int BAR_BYTES = 1024;
  static constexpr int NSTAGE_RAW = (kSmemBudget - Z_BYTES - BAR_BYTES) / STAGE_BYTES;
  static constexpr int NSTAGE = NSTAGE_RAW > 8 ? 8 : NSTAGE_RAW;
  static constexpr int SMEM_BYTES = Z_BYTES + NSTAGE * STAGE_BYTES + BAR_BYTES + 1024;
  // drain chunking
  static constexpr int PC = (KR * NP <= 128) ? NP : 128 / KR;  // p columns per drain chunk
  static constexpr int OCH = (OT == 1) ? ((JR * OC <= 128) ? OC : 128 / JR) : 32;
  static constexpr int VW = (OT == 1) ? (JR < 8 ? JR : 8) : 8;  // elements per vector store

  static_assert(NB2 % G == 0, "G must divide nb2");
  static_assert((G * IN2) % NB1 == 0, "group must cover whole R rows");
  static_assert(NP % 16 == 0 && NP <= 256, "MMA N (R stage) must be a multiple of 16 <= 256");
  static_assert(IN1 % 16 == 0 && IN2 % 16 == 0, "block K must be a multiple of 16");
  static_assert(OUT2 % OC == 0 && OC % 16 == 0, "MMA N (L stage)");
  static_assert(NB1 % KR == 0, "R rounds");
  static_assert(KR % 8 == 0 || (KR == NB1 && 8 % NB1 == 0), "16-byte Z chunks");
  static_assert(G % JR == 0, "L rounds");
  static_assert(NP % PC == 0 && PC % 8 == 0 && (KR * PC) % 8 == 0, "drain chunk");
  static_assert(OT == 0 || (VW == 8 || VW == 4 || VW == 2), "output vector width");
  static_assert(OT == 1 || (OC % 32 == 0), "flat output chunks");
  static_assert(NSTAGE >= 2, "shared memory");
  static_assert(LPS >= 1, "L slice larger than a stage");
};

template <class C>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmR,
                  const __grid_constant__ CUtensorMap tmL, __nv_bfloat16* __restrict__ Y,
                  int64_t rows, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* zbuf = smem;                                  // Z tile, 1024-aligned
  uint8_t* ring = smem + C::Z_BYTES;                     // NSTAGE stages, 1024-aligned
  Bars* bars = (Bars*)(ring + C::NSTAGE * C::STAGE_BYTES);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t ntiles = (rows + C::BM - 1) / C::BM;
  const int64_t nunits = ntiles * C::NGROUPS;
  const int group = blockIdx.x % C::NGROUPS;  // gridDim.x is a multiple of NGROUPS

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      ptx::mbar_init(&bars->full[i], 1);
      ptx::mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->acc_full[i], 1);
      ptx::mbar_init(&bars->acc_empty[i], 4);
    }
    ptx::mbar_init(&bars->z_full, 4);
    ptx::mbar_init(&bars->z_empty, 1);
    ptx::mbar_init(&bars->mma_done, 1);
    bars->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&bars->tmem_base, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      ptx::tma_prefetch_desc(&tmX);
      ptx::tma_prefetch_desc(&tmR);
      ptx::tma_prefetch_desc(&tmL);
      const uint64_t pol_stream = ptx::policy_evict_normal();  // X is read by NGROUPS CTAs
      const uint64_t pol_keep = ptx::policy_evict_last();
      uint32_t it = 0;  // global stage counter
      bool ok = true;
      for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
        const int row0 = (int)((u / C::NGROUPS) * C::BM);
        // R stage: one X box + the R slices of its (up to 4) K steps per stage
        for (int b = 0; b < C::NXB && ok; ++b, ++it) {
          const int st = it % C::NSTAGE;
          const uint32_t ph = (it / C::NSTAGE) & 1;
          if (!wait_or_abort(&bars->empty[st], ph ^ 1, &bars->abort_flag, status)) { ok = false; break; }
          uint8_t* sbase = ring + st * C::STAGE_BYTES;
          int nk = 0;
          for (int t = 0; t < 4; ++t) nk += (b * 64 + t * 16 < C::N_IN) ? 1 : 0;
          ptx::mbar_arrive_expect_tx(&bars->full[st], C::XBOX_BYTES + nk * C::RPIECE);
          ptx::tma_load_2d(sbase, &tmX, &bars->full[st], b * 64, row0, pol_stream);
          for (int t = 0; t < nk; ++t) {
            const int col = b * 64 + t * 16;
            const int k = col / C::IN1, s = (col % C::IN1) / 16;
            ptx::tma_load_2d(sbase + C::XBOX_BYTES + t * C::RPIECE, &tmR, &bars->full[st], s * 16,
                             k * C::OUT1 + group * C::NP, pol_keep);
          }
        }
        // L stage: LPS slices per stage, in round order
        for (int sp = 0; sp < C::NSTAGE2 && ok; ++sp, ++it) {
          const int st = it % C::NSTAGE;
          const uint32_t ph = (it / C::NSTAGE) & 1;
          if (!wait_or_abort(&bars->empty[st], ph ^ 1, &bars->abort_flag, status)) { ok = false; break; }
          uint8_t* sbase = ring + st * C::STAGE_BYTES;
          const int p0 = sp * C::LPS;
          const int np = (C::NPIECE2 - p0) < C::LPS ? (C::NPIECE2 - p0) : C::LPS;
          ptx::mbar_arrive_expect_tx(&bars->full[st], np * C::LPIECE);
          for (int t = 0; t < np; ++t) {
            // piece index -> (round, jj, s): round-major, then j, then K step
            const int pi = p0 + t;
            const int r2 = pi / (C::JR * C::KS2);
            const int rem = pi % (C::JR * C::KS2);
            const int jj = rem / C::KS2, s = rem % C::KS2;
            const int jloc = (r2 / C::NOC) * C::JR + jj;
            const int oc = r2 % C::NOC;
            const int j = group * C::G + jloc;
            ptx::tma_load_2d(sbase + t * C::LPIECE, &tmL, &bars->full[st], s * 16,
                             j * C::OUT2 + oc * C::OC, pol_keep);
          }
        }
      }
      // Teardown: make sure every load this thread issued has landed.
      const uint32_t issued = it;
      for (uint32_t k = (issued > (uint32_t)C::NSTAGE ? issued - C::NSTAGE : 0); k < issued; ++k) {
        const int st = k % C::NSTAGE;
        ptx::mbar_wait_bounded(&bars->full[st], (k / C::NSTAGE) & 1, kWaitLimitNs);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = make_idesc(C::BM, C::NP);
      const uint32_t idesc2 = make_idesc(C::BM, C::OC);
      const uint32_t ring_s = ptx::smem_u32(ring);
      const uint32_t z_s = ptx::smem_u32(zbuf);
      uint32_t it = 0;     // ring stage counter
      uint32_t rnd = 0;    // accumulator round counter
      uint32_t unit_n = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++unit_n) {
        // ---- R stage
        int cur_box = -1;
        for (int r1 = 0; r1 < C::NR1 && ok; ++r1, ++rnd) {
          const int slot = rnd & 1;
          if (!wait_or_abort(&bars->acc_empty[slot], ((rnd >> 1) & 1) ^ 1, &bars->abort_flag, status)) { ok = false; break; }
          ptx::tc_fence_after();
          for (int kk = 0; kk < C::KR && ok; ++kk) {
            const int k = r1 * C::KR + kk;
            for (int s = 0; s < C::KS1; ++s) {
              const int col = k * C::IN1 + s * 16;
              const int b = col / 64, t = (col % 64) / 16;
              if (b != cur_box) {
                if (cur_box >= 0) { ptx::mma_commit(&bars->empty[it % C::NSTAGE]); ++it; }
                cur_box = b;
                if (!wait_or_abort(&bars->full[it % C::NSTAGE], (it / C::NSTAGE) & 1, &bars->abort_flag, status)) { ok = false; break; }
                ptx::tc_fence_after();
              }
              const uint32_t sb = ring_s + (it % C::NSTAGE) * C::STAGE_BYTES;
              const uint64_t adesc = make_sdesc(sb + t * 32, 1024, 2);
              const uint64_t bdesc = make_sdesc(sb + C::XBOX_BYTES + t * C::RPIECE, 256, 6);
              ptx::mma_bf16_ss(tmem + slot * C::SLOT + kk * C::NP, adesc, bdesc, idesc1, s > 0 ? 1u : 0u);
            }
          }
          if (!ok) break;
          ptx::mma_commit(&bars->acc_full[slot]);
        }
        if (!ok) break;
        ptx::mma_commit(&bars->empty[it % C::NSTAGE]);  // release the last X box
        ++it;
        // ---- wait for the permuted Z tile
        if (!wait_or_abort(&bars->z_full, unit_n & 1, &bars->abort_flag, status)) { ok = false; break; }
        ptx::tc_fence_after();
        // ---- L stage
        int piece = 0;
        for (int r2 = 0; r2 < C::NR2 && ok; ++r2, ++rnd) {
          const int slot = rnd & 1;
          if (!wait_or_abort(&bars->acc_empty[slot], ((rnd >> 1) & 1) ^ 1, &bars->abort_flag, status)) { ok = false; break; }
          ptx::tc_fence_after();
          const int oc = r2 % C::NOC;
          for (int jj = 0; jj < C::JR && ok; ++jj) {
            const int jloc = (r2 / C::NOC) * C::JR + jj;
            for (int s = 0; s < C::KS2; ++s, ++piece) {
              if (piece % C::LPS == 0) {
                if (piece > 0) { ptx::mma_commit(&bars->empty[it % C::NSTAGE]); ++it; }
                if (!wait_or_abort(&bars->full[it % C::NSTAGE], (it / C::NSTAGE) & 1, &bars->abort_flag, status)) { ok = false; break; }
                ptx::tc_fence_after();
              }
              const uint32_t sb = ring_s + (it % C::NSTAGE) * C::STAGE_BYTES;
              const int zc = jloc * C::IN2 + s * 16;
              const uint64_t adesc = make_sdesc(z_s + (zc / 64) * (C::BM * 128) + (zc % 64) * 2, 1024, 2);
              const uint64_t bdesc = make_sdesc(sb + (piece % C::LPS) * C::LPIECE, 256, 6);
              ptx::mma_bf16_ss(tmem + slot * C::SLOT + jj * C::OC, adesc, bdesc, idesc2, s > 0 ? 1u : 0u);
            }
            (void)oc;
          }
          if (!ok) break;
          ptx::mma_commit(&bars->acc_full[slot]);
        }
        if (!ok) break;
        ptx::mma_commit(&bars->empty[it % C::NSTAGE]);  // release the last L stage
        ++it;
        ptx::mma_commit(&bars->z_empty);                 // Z may be overwritten
      }
      // Teardown: wait for every issued MMA before TMEM is freed.
      ptx::mma_commit(&bars->mma_done);
      wait_mma_done(&bars->mma_done, &bars->abort_flag, status);
    }
  } else {
    // ================================================================ TMEM drain (rows)
    const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;            // row within the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t z_s = ptx::smem_u32(zbuf);
    uint32_t rnd = 0, unit_n = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++unit_n) {
      const int64_t grow = (u / C::NGROUPS) * C::BM + r;
      // ---- R-stage rounds -> permuted bf16 Z tile in shared memory
      for (int r1 = 0; r1 < C::NR1 && ok; ++r1, ++rnd) {
        const int slot = rnd & 1;
        if (!wait_or_abort(&bars->acc_full[slot], (rnd >> 1) & 1, &bars->abort_flag, status)) { ok = false; break; }
        if (r1 == 0 && !wait_or_abort(&bars->z_empty, (unit_n & 1) ^ 1, &bars->abort_flag, status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t tbase = tmem + lane_off + slot * C::SLOT;
#pragma unroll 1
        for (int pc = 0; pc < C::NP; pc += C::PC) {
          float v[C::KR][C::PC];
#pragma unroll
          for (int kk = 0; kk < C::KR; ++kk) {
#pragma unroll
            for (int c8 = 0; c8 < C::PC; c8 += 8) {
              uint32_t rr[8];
              ptx::tmem_ld8(tbase + kk * C::NP + pc + c8, rr);
#pragma unroll
              for (int e = 0; e < 8; ++e) v[kk][c8 + e] = __uint_as_float(rr[e]);
            }
          }
          ptx::tmem_wait_ld();
          // 16-byte chunks of 8 consecutive flat columns; enumeration idx = p_rel*KR + k_rel
#pragma unroll
          for (int c = 0; c < (C::KR * C::PC) / 8; ++c) {
            const int idx0 = c * 8;
            const int t0 = (pc + idx0 / C::KR) * C::NB1 + r1 * C::KR + idx0 % C::KR;  // local flat column
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i0 = idx0 + 2 * e, i1 = i0 + 1;
              w[e] = ptx::pack_bf16x2(v[i0 % C::KR][i0 / C::KR], v[i1 % C::KR][i1 / C::KR]);
            }
            const uint32_t chunk = (uint32_t)((t0 % 64) / 8);
            const uint32_t addr = z_s + (t0 / 64) * (C::BM * 128) + (r / 8) * 1024 + (r % 8) * 128 +
                                  ((chunk ^ (uint32_t)(r % 8)) * 16);
            ptx::st_shared_v4(addr, w[0], w[1], w[2], w[3]);
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->acc_empty[slot]);
      }
      if (!ok) break;
      ptx::fence_proxy_async_smem();  // Z writes -> visible to the tensor cores
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->z_full);
      // ---- L-stage rounds -> Y
      for (int r2 = 0; r2 < C::NR2 && ok; ++r2, ++rnd) {
        const int slot = rnd & 1;
        if (!wait_or_abort(&bars->acc_full[slot], (rnd >> 1) & 1, &bars->abort_flag, status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t tbase = tmem + lane_off + slot * C::SLOT;
        const int jb = group * C::G + (r2 / C::NOC) * C::JR;  // first global j of the round
        const int ob = (r2 % C::NOC) * C::OC;                 // first o of the round
        __nv_bfloat16* yrow = Y + grow * (int64_t)C::N_OUT;
        const bool live = grow < rows;
        if (C::OT == 1) {
#pragma unroll 1
          for (int oc0 = 0; oc0 < C::OC; oc0 += C::OCH) {
            float v[C::JR][C::OCH];
#pragma unroll
            for (int jj = 0; jj < C::JR; ++jj) {
#pragma unroll
              for (int c8 = 0; c8 < C::OCH; c8 += 8) {
                uint32_t rr[8];
                ptx::tmem_ld8(tbase + jj * C::OC + oc0 + c8, rr);
#pragma unroll
                for (int e = 0; e < 8; ++e) v[jj][c8 + e] = __uint_as_float(rr[e]);
              }
            }
            ptx::tmem_wait_ld();
            if (live) {
#pragma unroll
              for (int oo = 0; oo < C::OCH; ++oo) {
                const int o = ob + oc0 + oo;
#pragma unroll
                for (int jv = 0; jv < C::JR; jv += C::VW) {
                  __nv_bfloat16* dst = yrow + (int64_t)o * C::NB2 + jb + jv;
                  if (C::VW == 8) {
                    ptx::st_global_v4(dst, ptx::pack_bf16x2(v[jv][oo], v[jv + 1][oo]),
                                      ptx::pack_bf16x2(v[jv + 2][oo], v[jv + 3][oo]),
                                      ptx::pack_bf16x2(v[jv + 4][oo], v[jv + 5][oo]),
                                      ptx::pack_bf16x2(v[jv + 6][oo], v[jv + 7][oo]));
                  } else if (C::VW == 4) {
                    ptx::st_global_v2(dst, ptx::pack_bf16x2(v[jv][oo], v[jv + 1][oo]),
                                      ptx::pack_bf16x2(v[jv + 2][oo], v[jv + 3][oo]));
                  } else {
                    *(uint32_t*)dst = ptx::pack_bf16x2(v[jv][oo], v[jv + 1][oo]);
                  }
                }
              }
            }
          }
        } else {
          // y[j*out2 + o]: one j per round (JR == 1 when out2 > 256) or JR whole blocks
#pragma unroll 1
          for (int jj = 0; jj < C::JR; ++jj) {
#pragma unroll 1
            for (int oc0 = 0; oc0 < C::OC; oc0 += 32) {
              uint32_t rr[32];
#pragma unroll
              for (int c8 = 0; c8 < 32; c8 += 8) {
                uint32_t t8[8];
                ptx::tmem_ld8(tbase + jj * C::OC + oc0 + c8, t8);
#pragma unroll
                for (int e = 0; e < 8; ++e) rr[c8 + e] = t8[e];
              }
              ptx::tmem_wait_ld();
              if (live) {
                __nv_bfloat16* dst = yrow + (int64_t)(jb + jj) * C::OUT2 + ob + oc0;
#pragma unroll
                for (int c8 = 0; c8 < 32; c8 += 8) {
                  ptx::st_global_v4(dst + c8,
                                    ptx::pack_bf16x2(__uint_as_float(rr[c8]), __uint_as_float(rr[c8 + 1])),
                                    ptx::pack_bf16x2(__uint_as_float(rr[c8 + 2]), __uint_as_float(rr[c8 + 3])),
                                    ptx::pack_bf16x2(__uint_as_float(rr[c8 + 4]), __uint_as_float(rr[c8 + 5])),
                                    ptx::pack_bf16x2(__uint_as_float(rr[c8 + 6]), __uint_as_float(rr[c8 + 7])));
                }
              }
            }
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->acc_empty[slot]);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

template <class C>
static cudaError_t launch_tc_fwd(const void* X, const void* R, const void* L, void* Y,
                                 const Shape& s, int* status, cudaStream_t st) {
  if (s.rows == 0) return cudaSuccess;
  CUtensorMap mX, mR, mL;
  if (!make_map_2d(&mX, X, C::N_IN, (uint64_t)s.rows, 64, C::BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mR, R, C::IN1, (uint64_t)C::NB1 * C::OUT1, 16, C::NP, CU_TENSOR_MAP_SWIZZLE_32B) ||
      !make_map_2d(&mL, L, C::IN2, (uint64_t)C::NB2 * C::OUT2, 16, C::OC, CU_TENSOR_MAP_SWIZZLE_32B))
    return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = ensure_smem_attr((const void*)tc_fwd_kernel<C>, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int64_t nunits = ((s.rows + C::BM - 1) / C::BM) * C::NGROUPS;
  int64_t grid = (num_sms() / C::NGROUPS) * C::NGROUPS;
  const int64_t units_rounded = ((nunits + C::NGROUPS - 1) / C::NGROUPS) * C::NGROUPS;
  if (grid > units_rounded) grid = units_rounded;
  if (grid < C::NGROUPS) grid = C::NGROUPS;
  return launch_kernel(tc_fwd_kernel<C>, dim3((unsigned)grid), dim3(kTcThreads), C::SMEM_BYTES, st, false,
                       mX, mR, mL, (__nv_bfloat16*)Y, s.rows, status);
}

// Instantiated shape (nb1, in1, out1, nb2, in2, out2, out_transpose, G).
using CfgNb4 = FwdCfg<4, 256, 256, 4, 256, 1024, 0, 1>;     // nblocks = 4, 1024 -> 4096

template <class C>
static bool shape_is(const Shape& s) {
  return s.nb1 == C::NB1 && s.in1 == C::IN1 && s.out1 == C::OUT1 && s.nb2 == C::NB2 &&
         s.in2 == C::IN2 && s.out2 == C::OUT2 && s.out_transpose == C::OT;
}

bool tc_fwd_supported(const Shape& s) {
  return shape_is<CfgNb4>(s);
}

cudaError_t tc_fwd(const void* X, const void* R, const void* L, void* Y, const Shape& s,
                   int* status, cudaStream_t st) {
  if (shape_is<CfgNb4>(s)) return launch_tc_fwd<CfgNb4>(X, R, L, Y, s, status, st);
  return cudaErrorNotSupported;
}

}  // namespace monarch
