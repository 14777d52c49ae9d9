// One block-diagonal stage of a Monarch map, weights resident in shared memory:
//
//   out[r][col(b, p)] = sum_i in[r][b*IN + i] * W[b][p][i],     b < NB, p < OUT, i < IN
//   col(b, p) = p*NB + b   (OT = 1: the per-row (NB x OUT) -> (OUT x NB) transpose, i.e. the
//                           permutation P of the Monarch factorisation, or P_out)
//             = b*OUT + p  (OT = 0: block-contiguous)
//
// For the 64 x 64-block shapes (n = 4096) the middle vector of a row tile does not fit on chip,
// so the forward is two of these stages through a middle buffer: Z = P blockdiag(R) x, then
// y = P_out blockdiag(L) Z.  Folding each permutation into the stage that produces its input
// replaces the separate row-transpose passes (a full read and write of the activations each).
//
// The blocks are taken in rounds of 16.  Each CTA owns a group of RG consecutive rounds for the
// whole launch and keeps those rounds' weights in shared memory (64 x 64 blocks: one round,
// 128 KB); the CTAs of a group split the 64-row units of the input between them.  Per unit and
// round the input columns of the round arrive as 64-column TMA boxes (128B swizzle) in a deep
// ring; M = 64 MMAs put blocks 0..7 of the round at TMEM lane offset 0 and 8..15 at lane offset
// 16 (the two halves of the M = 64 data-path layout), so a drain thread owns one row and 8
// consecutive blocks.  The drain rounds to bf16.  With OT = 1 a round's output for one row and
// one output column p is 16 consecutive blocks, a 32-byte piece of the row (the rest belongs
// to the other rounds), so the drain stages chunks of 8 output columns x 64 rows in shared
// memory, laid out [p][row][16 blocks] so that a warp's 16-byte stores are contiguous, and
// one thread writes each chunk with a 3-D TMA store whose inner rows are those 32-byte pieces
// (TMA moves such pieces about 1.4x faster than 16-byte stores from registers, and
// asynchronously); the accumulators are released as soon as they are read.  With OT = 0 the
// drain stores 16-byte chunks of block-contiguous rows from registers.  A round's
// accumulators take 8*OUT TMEM columns; two slots alternate when they fit (OUT <= 32), else one.
// Roles: warp 0 TMA producer, warp 1 MMA issuer and TMEM owner, warps 2..9 drain (two per TMEM
// lane quadrant, each taking half of the OUT columns).  All waits are bounded.
#include "tc_common.cuh"

namespace monarch {

constexpr int kStageThreads = 320;  // 10 warps
constexpr int kStageDrainWarps = 8;

template <int NB_, int IN_, int OUT_, int OT_, int RG_>
struct StageCfg {
  static constexpr int NB = NB_, IN = IN_, OUT = OUT_, OT = OT_;
  static constexpr int BM = 64;
  static constexpr int N_IN = NB * IN, N_OUT = NB * OUT;
  static constexpr int KS = IN / 16;            // K steps of 16 per block
  static constexpr int NR = NB / 16;            // rounds of 16 blocks
  static constexpr int RG = RG_;                // rounds per CTA group (weights resident)
  static constexpr int NG = NR / RG;            // groups
  static constexpr int BPR = IN / 4;            // 64-column boxes per round (16 blocks x IN)
  static constexpr int SLOT = 8 * OUT;          // TMEM columns per round
  static constexpr int NSLOT = 2 * SLOT <= 512 ? 2 : 1;
  static constexpr int TMEM_COLS = NSLOT * SLOT <= 32 ? 32 : (NSLOT * SLOT <= 64 ? 64 : (NSLOT * SLOT <= 128 ? 128 : (NSLOT * SLOT <= 256 ? 256 : 512)));
  static constexpr int WPIECE = OUT * 32;       // one block's OUT rows x 16 K values, 32B swizzle
  static constexpr int W_BYTES = RG * 16 * KS * WPIECE;
  static constexpr int XBOX = BM * 128;         // 64 rows x 64 bf16
  static constexpr int OCHUNK = 8 * BM * 32;    // OT = 1 staging: 8 output columns x 64 rows x 16 blocks
  static constexpr int STG_BYTES = OT == 1 ? 2 * OCHUNK : 0;  // one chunk buffer per drain group
  static constexpr int NSTAGE_RAW = (kSmemBudget - W_BYTES - STG_BYTES - 1024) / XBOX;
  static constexpr int NSTAGE = NSTAGE_RAW > 16 ? 16 : NSTAGE_RAW;
  static constexpr int SMEM_BYTES = W_BYTES + STG_BYTES + NSTAGE * XBOX + 1024 + 1024;
  static constexpr int P_HALF = OUT / 2;        // output columns per drain warp
  // Blocks never straddle a 64-column box, so the boxes of a round (and the rounds of a group)
  // may be taken in any order: each CTA starts at its own box and round.
  static constexpr bool STAGGER = 64 % IN == 0;
  static_assert(NB % 16 == 0 && NR % RG == 0, "rounds of 16 blocks, whole groups");
  static_assert(IN % 16 == 0 && OUT % 16 == 0 && SLOT <= 512, "block sizes");
  static_assert(N_IN % 64 == 0 && (16 * IN) % 64 == 0, "64-column boxes align with rounds");
  static_assert(WPIECE % 256 == 0, "32B-swizzle atoms");
  static_assert(NSTAGE >= 4, "shared memory");
};

struct StageBars {
  uint64_t full[16], empty[16];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

// This CTA's group and its place among the group's CTAs (the grid is a multiple of NG).
template <class C>
__device__ __forceinline__ int stage_group() { return (int)(blockIdx.x % C::NG); }
template <class C>
__device__ __forceinline__ int64_t stage_first_unit() { return blockIdx.x / C::NG; }
template <class C>
__device__ __forceinline__ int64_t stage_unit_step() { return gridDim.x / C::NG; }
// Round of the group (0..RG-1) taken r-th by this CTA, and box taken j-th within a round.
template <class C>
__device__ __forceinline__ int stage_round(int r) {
  return C::STAGGER ? (int)((r + blockIdx.x / C::NG) % C::RG) : r;
}
template <class C>
__device__ __forceinline__ int stage_box(int j) {
  return C::STAGGER ? (int)((j + blockIdx.x / C::NG / C::RG) % C::BPR) : j;
}

template <class C>
__global__ void __launch_bounds__(kStageThreads, 1)
    tc_stage_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmO,
                    const __nv_bfloat16* __restrict__ W, __nv_bfloat16* __restrict__ out, int64_t rows,
                    int w_is_input, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* wsm = smem;                        // resident weights
  uint8_t* stg = smem + C::W_BYTES;           // OT = 1 output chunks
  uint8_t* ring = stg + C::STG_BYTES;         // input boxes
  StageBars* bars = (StageBars*)(ring + C::NSTAGE * C::XBOX);
  int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t nunits = (rows + C::BM - 1) / C::BM;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      ptx::mbar_init(&bars->full[i], 1);
      ptx::mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->acc_full[i], 1);
      ptx::mbar_init(&bars->acc_empty[i], kStageDrainWarps);
    }
    ptx::mbar_init(&bars->mma_done, 1);
    bars->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  // Weights that are a caller input (R, L) do not depend on the previous kernel of the stream:
  // they are copied in before the grid-dependency wait.  Weights made by an earlier kernel of
  // the same call (the transposed factors) only after it.  Piece (b, s) holds rows p < OUT of
  // W[b], K values [16 s, 16 s + 16), 32B-swizzled K-major: chunk c of row n lands at
  // n*32 + ((c ^ ((n >> 2) & 1)) << 4).
  if (!w_is_input) ptx::griddep_wait();
  {
    const uint32_t w_s = ptx::smem_u32(wsm);
    const int b_first = stage_group<C>() * C::RG * 16;  // first block of this CTA's group
    for (int g = threadIdx.x; g < C::RG * 16 * C::KS * C::OUT * 2; g += kStageThreads) {
      const int c = g & 1, n = (g >> 1) % C::OUT, piece = (g >> 1) / C::OUT;
      const int b = b_first + piece / C::KS, s = piece % C::KS;
      ptx::cp_async_16(w_s + piece * C::WPIECE + n * 32 + ((c ^ ((n >> 2) & 1)) << 4),
                       W + ((int64_t)b * C::OUT + n) * C::IN + s * 16 + c * 8);
    }
    ptx::cp_async_wait_all();
    ptx::fence_proxy_async_smem();  // written by the generic proxy, read by the tensor cores
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      ptx::tma_prefetch_desc(&tmA);
      const uint64_t pol = ptx::policy_evict_first();
      uint32_t it = 0;
      bool ok = true;
      const int r0 = stage_group<C>() * C::RG;
      for (int64_t u = stage_first_unit<C>(); u < nunits && ok; u += stage_unit_step<C>()) {
        const int row0 = (int)(u * C::BM);
        for (int q = 0; q < C::RG * C::BPR; ++q, ++it) {
          const int st = it % C::NSTAGE;
          const int b = (r0 + stage_round<C>(q / C::BPR)) * C::BPR + stage_box<C>(q % C::BPR);
          if (!wait_or_abort(&bars->empty[st], ((it / C::NSTAGE) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(&bars->full[st], C::XBOX);
          ptx::tma_load_2d(ring + st * C::XBOX, &tmA, &bars->full[st], b * 64, row0, pol);
        }
      }
      const uint32_t issued = it;
      for (uint32_t k = (issued > (uint32_t)C::NSTAGE ? issued - C::NSTAGE : 0); k < issued; ++k)
        ptx::mbar_wait_bounded(&bars->full[k % C::NSTAGE], (k / C::NSTAGE) & 1, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer (whole warp)
    constexpr uint32_t idesc = make_idesc(C::BM, C::OUT);
    const uint64_t ring_a = make_sdesc(ptx::smem_u32(ring), 1024, 2);  // 128B swizzle
    const uint64_t w_b = make_sdesc(ptx::smem_u32(wsm), 256, 6);       // 32B swizzle
    uint32_t it = 0, rnd = 0;
    bool ok = true;
    for (int64_t u = stage_first_unit<C>(); u < nunits && ok; u += stage_unit_step<C>()) {
      for (int rr = 0; rr < C::RG && ok; ++rr, ++rnd) {
        const int rl = stage_round<C>(rr);  // round within the group: weight pieces rl*16*KS ...
        const int slot = C::NSLOT == 2 ? (int)(rnd & 1) : 0;
        const uint32_t use = C::NSLOT == 2 ? rnd >> 1 : rnd;  // uses of this slot so far
        if (!warp_wait_or_abort(lane, &bars->acc_empty[slot], (use & 1) ^ 1, abort_flag, status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t dslot = tmem + slot * C::SLOT;
        for (int j = 0; j < C::BPR; ++j, ++it) {
          const int bb = stage_box<C>(j);
          const int st = it % C::NSTAGE;
          if (!warp_wait_or_abort(lane, &bars->full[st], (it / C::NSTAGE) & 1, abort_flag, status)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint64_t soff = (uint64_t)((st * C::XBOX) >> 4);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int c = bb * 64 + 16 * t;  // column within the round
            const int kk = c / C::IN, s = (c % C::IN) / 16;
            const uint32_t d = dslot + ((uint32_t)(kk >> 3) << 20) + (uint32_t)((kk & 7) * C::OUT);
            const int piece = (rl * 16 + kk) * C::KS + s;
            ptx::mma_bf16_ss_elect(d, ring_a + soff + (uint64_t)((32 * t) >> 4),
                                   w_b + (uint64_t)((piece * C::WPIECE) >> 4), idesc, s > 0 ? 1u : 0u);
          }
          ptx::mma_commit_elect(&bars->empty[st]);  // the box is free once these MMAs finish
        }
        if (!ok) break;
        ptx::mma_commit_elect(&bars->acc_full[slot]);
      }
    }
    ptx::mma_commit_elect(&bars->mma_done);
    if (lane == 0) wait_mma_done(&bars->mma_done, abort_flag, status);
    __syncwarp();
  } else {
    // ================================================================ drain (8 warps)
    const int quad = warp & 3;              // TMEM lane quadrant of this warp
    const int ph = (warp - 2) >> 2;         // drain group: which half of the OUT columns
    const int half = lane >> 4;             // lane offset 0 / 16 -> blocks 0..7 / 8..15 of a round
    const int r = quad * 16 + (lane & 15);  // row within the 64-row unit
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool leader = (warp & 3) == 2 && lane == 0;  // warps 2 and 6 lead their groups
    const uint32_t buf = ptx::smem_u32(stg) + (uint32_t)(ph * C::OCHUNK);
    uint32_t rnd = 0;
    bool ok = true;
    const int r0 = stage_group<C>() * C::RG;
    for (int64_t u = stage_first_unit<C>(); u < nunits && ok; u += stage_unit_step<C>()) {
      const int64_t row = u * C::BM + r;
      const bool live = row < rows;
      __nv_bfloat16* orow = out + (live ? row : 0) * C::N_OUT;
      for (int rr = 0; rr < C::RG && ok; ++rr, ++rnd) {
        const int r1 = r0 + stage_round<C>(rr);
        const int slot = C::NSLOT == 2 ? (int)(rnd & 1) : 0;
        const uint32_t use = C::NSLOT == 2 ? rnd >> 1 : rnd;
        if (!wait_or_abort(&bars->acc_full[slot], use & 1, abort_flag, status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t tb = tmem + lane_off + slot * C::SLOT;
        const int b0 = r1 * 16 + half * 8;  // first of this thread's 8 blocks
#pragma unroll 1
        for (int pc = ph * C::P_HALF; pc < (ph + 1) * C::P_HALF; pc += 8) {
          float v[8][8];
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            uint32_t rr[8];
            ptx::tmem_ld8(tb + kk * C::OUT + pc, rr);
#pragma unroll
            for (int e = 0; e < 8; ++e) v[kk][e] = __uint_as_float(rr[e]);
          }
          ptx::tmem_wait_ld();
          if (pc + 8 == (ph + 1) * C::P_HALF) {
            // this warp has read all its accumulator columns of the round: release them
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars->acc_empty[slot]);
          }
          if (C::OT == 1) {
            // the group's previous chunk store must have read the buffer before it is rewritten
            if (leader) ptx::bulk_wait_read_all();
            ptx::named_bar_sync(1 + ph, 128);
#pragma unroll
            for (int e = 0; e < 8; ++e)  // chunk layout [p][row][16 blocks]
              ptx::st_shared_v4(buf + (uint32_t)(e * (C::BM * 32) + r * 32 + half * 16),
                                ptx::pack_bf16x2(v[0][e], v[1][e]), ptx::pack_bf16x2(v[2][e], v[3][e]),
                                ptx::pack_bf16x2(v[4][e], v[5][e]), ptx::pack_bf16x2(v[6][e], v[7][e]));
            ptx::fence_proxy_async_smem();
            ptx::named_bar_sync(1 + ph, 128);
            if (leader) {  // out[row][(pc + e)*NB + 16 r1 + (0..15)]; rows past the end are clipped
              ptx::tma_store_3d(&tmO, stg + ph * C::OCHUNK, r1 * 16, (int)(u * C::BM), pc);
              ptx::bulk_commit_group();
            }
          } else if (live) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // out[(b0 + kk)*OUT + pc .. + 8]
              *(uint4*)(orow + (b0 + kk) * C::OUT + pc) =
                  make_uint4(ptx::pack_bf16x2(v[kk][0], v[kk][1]), ptx::pack_bf16x2(v[kk][2], v[kk][3]),
                             ptx::pack_bf16x2(v[kk][4], v[kk][5]), ptx::pack_bf16x2(v[kk][6], v[kk][7]));
          }
        }
      }
    }
    if (C::OT == 1 && leader) ptx::bulk_wait_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

template <class C>
static cudaError_t launch_stage(const void* A, const void* W, bool w_is_input, void* out, int64_t rows,
                                int* status, cudaStream_t st, bool pdl) {
  if (rows == 0) return cudaSuccess;
  CUtensorMap mA, mO;
  if (!make_map_2d(&mA, A, C::N_IN, (uint64_t)rows, 64, C::BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  mO = mA;
  if (C::OT == 1) {
    // out viewed as (block k < NB, row, output column p < OUT): out[row][p*NB + k]
    const uint64_t dims[3] = {(uint64_t)C::NB, (uint64_t)rows, (uint64_t)C::OUT};
    const uint64_t strides[2] = {(uint64_t)C::N_OUT * 2, (uint64_t)C::NB * 2};
    const uint32_t box[3] = {16, (uint32_t)C::BM, 8};
    if (!make_map_3d(&mO, out, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE)) return cudaErrorInvalidValue;
  }
  cudaError_t e = ensure_smem_attr((const void*)tc_stage_kernel<C>, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // NG groups of CTAs, as many CTAs per group as fill the SMs (at most one per unit)
  const int64_t nunits = (rows + C::BM - 1) / C::BM;
  int64_t per = num_sms() / C::NG;
  if (per < 1) per = 1;
  if (per > nunits) per = nunits;
  return launch_kernel(tc_stage_kernel<C>, dim3((unsigned)(per * C::NG)), dim3(kStageThreads), C::SMEM_BYTES, st,
                       pdl, mA, mO, (const __nv_bfloat16*)W, (__nv_bfloat16*)out, rows, w_is_input ? 1 : 0,
                       status);
}

// ---------------------------------------------------------------- shapes
// 64 blocks of 64 x 64 per factor (n = 4096): one round per CTA group, 128 KB of weights each.
using Stage64T = StageCfg<64, 64, 64, 1, 1>;
using Stage64N = StageCfg<64, 64, 64, 0, 1>;
// 768 -> 3072 (R: 16 blocks of 48 x 48; L: 48 blocks of 64 x 16): every factor fits resident.
// Its backward's Z and dU passes use stages; its forward stays the fused row-tile kernel, which
// measured faster than two stages (32.8 vs 35.8 us for 8192 rows).
using StageR768 = StageCfg<16, 48, 48, 1, 1>;   // Z = P blockdiag(R) X
using StageLt768 = StageCfg<48, 64, 16, 1, 3>;  // dU = P^-1 blockdiag(L^T) dV

static bool is_sq64(const Shape& s) { return tc_split_supported(s) && s.nb1 == 64; }
static bool is_r768(const Shape& s) {
  return s.nb1 == 16 && s.in1 == 48 && s.out1 == 48 && s.nb2 == 48 && s.in2 == 16 && s.out2 == 64 &&
         s.out_transpose == 1;
}

bool tc_stage_supported(const Shape& s) { return is_sq64(s) || is_r768(s); }
// Shapes whose workspace forward is the two stages (R, then L).
bool tc_stage_fwd_supported(const Shape& s) { return is_sq64(s); }

// One stage of a tc_stage_supported shape (see StageKind in common.cuh).
cudaError_t tc_stage(const void* A, const void* W, void* out, StageKind k, const Shape& s, int* status,
                     cudaStream_t st, bool pdl, bool w_early) {
  const bool input = w_early;
  if (is_sq64(s)) {
    const bool ot = k == StageKind::R || k == StageKind::Lt || (k == StageKind::L && s.out_transpose == 1);
    return ot ? launch_stage<Stage64T>(A, W, input, out, s.rows, status, st, pdl)
              : launch_stage<Stage64N>(A, W, input, out, s.rows, status, st, pdl);
  }
  if (is_r768(s)) {
    switch (k) {
      case StageKind::R: return launch_stage<StageR768>(A, W, input, out, s.rows, status, st, pdl);
      case StageKind::Lt: return launch_stage<StageLt768>(A, W, input, out, s.rows, status, st, pdl);
      default: return cudaErrorNotSupported;
    }
  }
  return cudaErrorNotSupported;
}

// Y = X M^T as two stages through the caller's middle buffer Z (rows x n_mid bf16), for the
// tc_stage_fwd_supported shapes.
cudaError_t tc_stage_fwd(const void* X, const void* R, const void* L, void* Y, void* Z, const Shape& s,
                         int* status, cudaStream_t st) {
  cudaError_t e = tc_stage(X, R, Z, StageKind::R, s, status, st, false, true);
  if (e != cudaSuccess) return e;
  return tc_stage(Z, L, Y, StageKind::L, s, status, st, true, true);
}

}  // namespace monarch
