// BF16 weight-gradient GEMMs on a pair of SMs (tcgen05.mma.cta_group::2), K-grouped:
// dW[e] = A_e^T B_e with the contraction over expert e's rows (A_e [n_e, M] and
// B_e [n_e, N] are MN-major: their rows are the K dimension).
//
// Pages: "Efficient MoE training for biological foundation models" (news.bpdata.com
// section 3: the backward of the fused GroupedLinear chain, whose weight gradients are
// grouped GEMMs over each expert's tokens).
//
// A 2-CTA cluster computes 256 x 256 tiles of dW[e]: each CTA loads the 128 M columns of
// A it owns and its half (128 columns) of B, 128 K rows per stage (one TMA copy of two
// 64-column chunks per operand, [chunk][k row] in shared memory), and the leader issues
// M=256, N=256, K=16 MMAs with both operands MN-major. Tiles are handed out longest
// expert first; an expert without rows gets zero gradients.
//
// The last k-block of an expert is ragged: its rows past n_e belong to the next expert
// and must not contribute. The leader issues only the MMA steps that hold the expert's
// rows, and inside the last partial 16-row step both CTAs zero their own rows past n_e.
// A CTA can zero its rows only after its own copy has landed, and 2-SM copies complete
// on the leader's barrier alone, so for that one stage per tile both CTAs load with the
// 1-SM form onto their own barriers; the second CTA (its otherwise idle warp 1) zeroes
// and then signals the leader's `rready` barrier with a remote arrive, and the leader's
// MMA thread zeroes its own rows and waits for `rready` before its MMAs.
#pragma once
#include "grouped_gemm_sm100.cuh"

namespace moe {

namespace kp {
constexpr int BM = 256;                       // M of a pair tile (128 per CTA)
constexpr int BMC = 128;
constexpr int BN = 256;                       // N of a pair tile (128 per CTA)
constexpr int BK = 128;                       // K rows per stage
constexpr int kStages = 3;
constexpr int kThreads = 384;
constexpr int kChunkBytes = 128 * 64 * 2;     // 64 columns x 128 k rows, 16 KB
constexpr int kABytes = 2 * kChunkBytes;      // this CTA's 128 columns of A
constexpr int kBBytes = 2 * kChunkBytes;      // this CTA's 128 columns of B
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kMaxE = 1024;
constexpr int kTmemCols = 512;
constexpr int kStgBytes = 32 * 64;            // an epilogue warp's staging tile: 32 rows x 32 bf16
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 8 * kStgBytes + 1024 + 3 * (kMaxE + 1) * 4;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
}  // namespace kp

// Epilogue of one dW tile for one warp: its 32 rows (m_row0.. of dW[e]) x this half's 128
// columns, in 32-column strips: tensor memory -> bf16 -> the warp's staging tile (64-byte
// swizzle: 16-byte chunk j of row r at r*64 + 16*(j ^ ((r>>1)&3))) -> one TMA store per
// strip, issued and waited on by lane 0 (a strip reuses the tile once the previous
// store has read it). Each lane storing its own row 16 bytes at a time made 32 separate
// L2 requests per instruction, which held back the tiles of experts with few rows. A
// strip that is not wholly inside [M, N) of dW[e] is stored by the lanes instead.
__device__ __forceinline__ void kp_wgrad_epilogue(const GemmParams& p, const CUtensorMap* tmO, uint8_t* stg,
                                                  const TileInfo& ti, uint32_t t_row, int half, int m_row0, int lane) {
  const bool zero = (ti.num_kb == 0);
  const int n0 = ti.n_blk * kp::BN;
  const int m = m_row0 + lane;
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
#pragma unroll 1
  for (int s = 0; s < 4; ++s) {
    const int c = half * (kp::BN / 2) + 32 * s;
    uint32_t v0[16], v1[16];
    tmem_ld_32x32b_x16(t_row + c, v0);
    tmem_ld_32x32b_x16(t_row + c + 16, v1);
    tmem_wait_ld();
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w[i] = zero ? 0u : pack_bf16x2(__uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1]));
      w[8 + i] = zero ? 0u : pack_bf16x2(__uint_as_float(v1[2 * i]), __uint_as_float(v1[2 * i + 1]));
    }
    const int col = n0 + c;
    if (col + 32 <= p.N && m_row0 + 32 <= p.M) {   // warp-uniform
      if (lane == 0) bulk_wait_group_read0();
      __syncwarp();
      uint8_t* row = stg + lane * 64;
      const int sw = (lane >> 1) & 3;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(row + 16 * (j ^ sw)) = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(tmO, stg, col, m_row0, ti.e);
        bulk_commit_group();
      }
    } else if (m < p.M) {
      __nv_bfloat16* o = out + (long long)ti.e * p.out_batch + (long long)m * p.ldo + col;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (col + 8 * j < p.N)
          *reinterpret_cast<uint4*>(o + 8 * j) = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
    }
  }
}

// Zero rows [valid, end) of the four 64-column chunks (A 2, B 2) of one stage of this
// CTA, one warp; then make the stores visible to the tensor cores' reads.
__device__ __forceinline__ void kp_zero_rows(uint8_t* a_st, uint8_t* b_st, int valid, int end, int lane) {
  const int zr = end - valid;
  if (zr > 0) {
    for (int i = lane; i < 4 * zr * 8; i += 32) {
      const int v = i & 7, rc = i >> 3;
      const int c = rc / zr, r = rc - c * zr;
      uint8_t* base = (c < 2) ? a_st + c * kp::kChunkBytes : b_st + (c - 2) * kp::kChunkBytes;
      *reinterpret_cast<uint4*>(base + (valid + r) * 128 + v * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  __syncwarp();
}

// tmA: A [R rows, M] as {64, R, M/64 chunks, 1}; tmB: B [R, N] as {64, R, N/64, 1};
// boxes {64, 128 k rows, 2 chunks, 1}. Output dW[e] [M, N] bf16 at p.out + e * p.out_batch;
// tmO: dW as {N, M, E}, boxes {32, 32, 1}, 64-byte swizzle.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kp::kThreads, 1)
    grouped_wgrad_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                   const __grid_constant__ CUtensorMap tmO, const GemmParams p) {
  using namespace kp;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kABytes;
  uint8_t* stg = smem + kStages * kStageBytes;   // 8 epilogue warps' staging tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg + 8 * kStgBytes);
  uint64_t* full = bars;                       // leader: 2-SM copies, and its own copies of a ragged stage
  uint64_t* empty = bars + kStages;            // both CTAs
  uint64_t* pfull = bars + 2 * kStages;        // second CTA: its own copies of a ragged stage
  uint64_t* rready = bars + 3 * kStages;       // leader: the second CTA has zeroed its ragged stage
  uint64_t* tfull = bars + 4 * kStages;        // both CTAs
  uint64_t* tempty = bars + 4 * kStages + 2;   // leader
  uint64_t* drained = bars + 4 * kStages + 4;  // second CTA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* row_off = reinterpret_cast<int32_t*>(stg + 8 * kStgBytes + 1024);
  int32_t* tile_off = row_off + (kMaxE + 1);
  int32_t* order = tile_off + (kMaxE + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int E = p.E;
  const int MT = (p.M + BM - 1) / BM, NT = (p.N + BN - 1) / BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&pfull[s], 1);
      mbar_init(&rready[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 16);   // 8 epilogue warps in each CTA of the pair
    }
    mbar_init(drained, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 3) {
    int carry_r = 0, carry_t = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int n = (e < E) ? p.split_sizes[e] : 0;
      const int tiles = (e < E) ? MT * NT : 0;
      int ir = n, it = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yr = __shfl_up_sync(0xffffffffu, ir, o);
        const int yt = __shfl_up_sync(0xffffffffu, it, o);
        if (lane >= o) {
          ir += yr;
          it += yt;
        }
      }
      if (e < E) {
        row_off[e] = carry_r + ir - n;
        tile_off[e] = carry_t + it - tiles;
      }
      carry_r += __shfl_sync(0xffffffffu, ir, 31);
      carry_t += __shfl_sync(0xffffffffu, it, 31);
    }
    if (lane == 0) {
      row_off[E] = carry_r;
      tile_off[E] = carry_t;
    }
  }
  if (warp == 2) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  rank_experts_by_rows(row_off, E, order);
  __syncthreads();
  cluster_sync();   // both CTAs' barriers are initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  TileWalker<true, BM> walk{row_off, tile_off, E, MT, NT, p.K, order};
  const int total = walk.total();
  auto stages_of = [](const TileInfo& ti) { return (ti.rows + BK - 1) / BK; };

  if (warp == 0) {
    // ---------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      ArmedRing ring, pring;   // leader: full; second CTA: its own ragged-stage barriers pfull
      bool ok = true;
      for (int t = pair; t < total && ok && !p.stall_loads; t += npairs) {
        const TileInfo ti = walk.decode(t);
        const int nk = stages_of(ti);
        // this CTA's 128 columns of A and of B, as 64-column chunk indices
        const int ca = ti.m_blk * (BM / 64) + 2 * (int)rank;
        const int cb = ti.n_blk * (BN / 64) + 2 * (int)rank;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          const int k0 = ti.row0 + kb * BK;
          if (kb < nk - 1 || (ti.rows % BK) == 0) {
            if (leader) {
              mbar_arrive_expect_tx(&full[stage], 2 * kStageBytes);
              ring.arm(stage, phase);
            }
            tma_load_4d_pair(sA + stage * kABytes, &tmA, &full[stage], 0, k0, ca, 0);
            tma_load_4d_pair(sB + stage * kBBytes, &tmB, &full[stage], 0, k0, cb, 0);
          } else {
            // ragged last stage: each CTA's copies land on its own barrier, so that it can
            // zero its rows past the expert before the MMAs read them
            uint64_t* bar = leader ? &full[stage] : &pfull[stage];
            mbar_arrive_expect_tx(bar, kStageBytes);
            (leader ? ring : pring).arm(stage, phase);
            tma_load_4d(sA + stage * kABytes, &tmA, bar, 0, k0, ca, 0);
            tma_load_4d(sB + stage * kBBytes, &tmB, bar, 0, k0, cb, 0);
          }
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // no copy may still be landing when either CTA leaves: the second CTA's own
      // ragged-stage copies complete on its pfull barriers, the rest on the leader's
      if (!leader && !ok) pring.drain(pfull, kStages, p.timeout_ns);
      pair_producer_drain(leader, ok, drained, p.timeout_ns, full, kStages, ring);
    }
  } else if (warp == 1 && !leader) {
    // -------------------- second CTA: zero its rows of each ragged stage, tell the leader
    const uint32_t rready_leader0 = map_to_rank(smem_u32(&rready[0]), 0);
    int stage = 0;
    uint32_t pmask = 0;   // phase parity of pfull per ring slot
    bool ok = true;
    for (int t = pair; t < total && ok; t += npairs) {
      const TileInfo ti = walk.decode(t);
      const int nk = stages_of(ti);
      for (int kb = 0; kb < nk; ++kb) {
        if (kb == nk - 1 && (ti.rows % BK) != 0) {
          if (!mbar_wait_bounded(&pfull[stage], (pmask >> stage) & 1u, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          pmask ^= 1u << stage;
          const int valid = ti.rows - kb * BK;
          kp_zero_rows(sA + stage * kABytes, sB + stage * kBBytes, valid, (valid + 15) / 16 * 16, lane);
          if (lane == 0) mbar_arrive_cluster(rready_leader0 + stage * 8);
        }
        if (++stage == kStages) stage = 0;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (pair leader)
    constexpr uint32_t idesc = make_idesc_bf16(BM, BN, true, true);
    int stage = 0;
    uint32_t phase = 0, rmask = 0;
    int lt = 0;
    bool ok = true;
    for (int t = pair; t < total && ok; t += npairs, ++lt) {
      const TileInfo ti = walk.decode(t);
      const int nk = stages_of(ti);
      const int acc = lt & 1;
      if (!mbar_wait_bounded<true>(&tempty[acc], ((lt >> 1) & 1) ^ 1, abort_flag, p.timeout_ns)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        int ksteps = BK / 16;
        if (kb == nk - 1 && (ti.rows % BK) != 0) {
          // MMAs only over the expert's rows; zero this CTA's rows inside the last partial
          // step, then wait until the second CTA has done the same with its rows
          const int valid = ti.rows - kb * BK;
          ksteps = (valid + 15) / 16;
          kp_zero_rows(sA + stage * kABytes, sB + stage * kBBytes, valid, ksteps * 16, lane);
          if (!mbar_wait_bounded<true>(&rready[stage], (rmask >> stage) & 1u, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          rmask ^= 1u << stage;
          tc_fence_after();
        }
        if (lane == 0) {
          const uint32_t a_addr = smem_u32(sA + stage * kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * kBBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            if (kk >= ksteps) break;
            // MN-major: 16 k rows = 2048 bytes; 64-column chunks kChunkBytes apart
            const uint64_t adesc = make_sdesc(a_addr + kk * 2048, kChunkBytes, 1024, 2);
            const uint64_t bdesc = make_sdesc(b_addr + kk * 2048, kChunkBytes, 1024, 2);
            mma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty[stage]);
        }
        __syncwarp();
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      // (an expert without rows: no MMAs, the commit arrives at once and the epilogue
      // writes zeros)
      if (lane == 0) mma_commit_pair(&tfull[acc]);
      __syncwarp();
    }
  } else if (warp >= 4) {
    // -------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r_local = q * 32 + lane;
    const uint32_t tempty_leader0 = map_to_rank(smem_u32(&tempty[0]), 0);
    int lt = 0;
    for (int t = pair; t < total; t += npairs, ++lt) {
      const TileInfo ti = walk.decode(t);
      const int acc = lt & 1;
      if (!mbar_wait_bounded(&tfull[acc], (lt >> 1) & 1, abort_flag, p.timeout_ns)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + acc * BN + ((uint32_t)(q * 32) << 16);
      kp_wgrad_epilogue(p, &tmO, stg + (warp - 4) * kStgBytes, ti, t_row, half,
                        ti.m_blk * BM + BMC * (int)rank + q * 32, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + acc * 8);
    }
    // the tile stores must have completed before the CTA (and its shared memory) goes
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // neither CTA leaves while the other can still signal it
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace moe
