// Grouped GEMM on a pair of SMs (tcgen05.mma.cta_group::2), BF16, M-grouped.
//
// A 2-CTA cluster computes 256 x 256 output tiles: each CTA loads its own 128 rows of A
// and its own half (128 columns) of B into its shared memory, the pair leader issues
// tcgen05.mma.cta_group::2 (M=256, N=256, K=16) that reads both CTAs' operands, and each
// CTA receives the 128 x 256 fp32 accumulator of its rows in its own tensor memory.
//
// A k-stage is 128 wide and each operand of a stage arrives with ONE TMA copy: the tensor
// maps view a matrix as 64-element (128-byte) chunks, so a box of two chunks x 128 rows
// lands as two canonical 128-byte-swizzled tiles back to back (K-major: [chunk][row];
// MN-major: [column chunk][k row]). Issuing a copy costs the TMA unit about the same
// whatever its size, so two 32 KB copies per 1024-cycle stage keep the tensor pipe fed
// where six 8-16 KB copies per 512-cycle stage did not. 3 stages of 64 KB per CTA.
//
// Synchronisation: both CTAs' TMA loads complete on the leader's `full` barrier (the
// 2-SM TMA form); the leader's MMA commits arrive on the `empty` and `tfull` barriers of
// both CTAs (multicast commit, no multicast loads); both CTAs' epilogue warps arrive on
// the leader's `tempty` barrier. Waits are bounded like in the 1-SM kernel.
//
// For fc1 the leader's half of B is the gate columns [n0, n0+128) and the other CTA's
// the up columns [F+n0, F+n0+128), so each CTA's accumulator holds [gate | up] for its
// rows and the ScaledSwiGLU epilogue stays thread-local.
//
// SwiGLU backward: warp 3 of each CTA copies the saved h of the rows being drained with
// TMA into a shared-memory ring of 32-column strips, ahead of the epilogue, which reads its
// row from there instead of one 16-byte global load per row and lane (as in the MXFP8
// pair kernel).
//
// Outputs: a warp whose 32 rows all belong to the tile's expert sends its bf16 results
// (STORE: the output; SwiGLU backward: dg and du) through a 2 KB shared-memory staging
// tile with one TMA store per 32x32 strip instead of 16-byte stores of 32 different rows
// per instruction; the other warps, the fused combine and fp32 outputs store per lane.
#pragma once
#include "grouped_gemm_sm100.cuh"

namespace moe {

namespace g2 {
constexpr int BM = 256;                       // rows of a pair tile
constexpr int BMC = 128;                      // rows per CTA
constexpr int BN = 256;
constexpr int BK = 128;                       // k per stage: two 64-element chunks
constexpr int kStages = 3;
constexpr int kThreads = 384;
constexpr int kABytes = BMC * BK * 2;         // 32 KB
constexpr int kBBytes = (BN / 2) * BK * 2;    // 32 KB: this CTA's half of B
constexpr int kChunkBytes = 128 * 64 * 2;     // one 64-element chunk of 128 rows (or k rows), 16 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kMaxE = 1024;
constexpr int kTmemCols = 512;
// SwiGLU backward: the saved h reaches the epilogue through shared memory, a two-slot
// ring of 32-column strips (g and u of the CTA's 128 rows, 64-byte swizzled: 16 KB) per
// column half; its 64 KB come out of the operand ring, which keeps two stages there.
constexpr int kHSlotBytes = 2 * 128 * 64;
constexpr int kHSlots = 2;
// STORE: a 2 KB staging tile (32 rows x 32 bf16) per epilogue warp for TMA stores
constexpr int kStgBytes = 32 * 64;
__host__ __device__ constexpr bool stages_h(int epi) { return epi == EPI_DSWIGLU; }
__host__ __device__ constexpr int stages_for(int epi) { return stages_h(epi) ? 2 : kStages; }
__host__ __device__ constexpr int side_bytes(int epi) {
  // SwiGLU backward: the h ring, then a staging tile per epilogue warp for dh
  return stages_h(epi) ? 2 * kHSlots * kHSlotBytes + 8 * kStgBytes : (epi == EPI_STORE ? 8 * kStgBytes : 0);
}
__host__ __device__ constexpr int smem_bytes(int epi) {
  return 1024 + stages_for(epi) * kStageBytes + side_bytes(epi) + 1024 + 2 * (kMaxE + 1) * 4;
}
constexpr int kSmemBytes = smem_bytes(EPI_STORE);
static_assert(smem_bytes(EPI_DSWIGLU) <= 232448 && smem_bytes(EPI_STORE) <= 232448, "shared memory per CTA");
}  // namespace g2

// STORE epilogue of one warp through TMA: its 32 rows (tile rows row0.., all inside the
// expert) x this half's 128 columns, in 32-column strips: tensor memory -> bf16 -> the
// warp's staging tile (64-byte swizzle: 16-byte chunk j of row r at r*64 +
// 16*(j ^ ((r>>1)&3))) -> one TMA store per strip by lane 0, which first waits until the
// previous strip's store has read the tile. A strip past N is stored by the lanes.
// Lane stores of 16 bytes per row made 32 separate L2 requests per instruction.
__device__ __forceinline__ void g2_store_tma(const GemmParams& p, const CUtensorMap* tmO, uint8_t* stg,
                                             const TileInfo& ti, uint32_t t_row, int half, long long row0,
                                             int lane) {
  const bool zero = (ti.num_kb == 0);
  const int n0 = ti.n_blk * g2::BN;
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
#pragma unroll 1
  for (int s = 0; s < 4; ++s) {
    const int c = half * (g2::BN / 2) + 32 * s;
    const int col = n0 + c;
    if (col >= p.N) break;   // warp-uniform; the rest of the half is past N too
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
    if (col + 32 <= p.N) {
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
        tma_store_3d(tmO, stg, col, (int)row0, 0);
        bulk_commit_group();
      }
    } else {
      __nv_bfloat16* o = out + (row0 + lane) * p.ldo + col;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (col + 8 * j < p.N)
          *reinterpret_cast<uint4*>(o + 8 * j) = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
    }
  }
}

// tmA: A [rows, K] as {64, rows, K/64 chunks, 1}; tmB: B_MN ? [E][K rows][N] as
// {64, K, N/64 chunks, E} : [E][N rows][K] as {64, N, K/64 chunks, E}; boxes {64, 128, 2, 1}.
// tmX: SwiGLU backward: the saved h [R, 2F] bf16 as {2F, R, 1}, box {32, 128}, 64-byte
// swizzle; STORE with p.tma_out: the output [R, N] bf16 as {N, R, 1}, box {32, 32},
// 64-byte swizzle; otherwise unused. tmY (SwiGLU backward only): dh [R, 2F] bf16 as
// {2F, R, 1}, box {32, 32}, 64-byte swizzle.
template <bool B_MN, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(g2::kThreads, 1)
    grouped_gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                  const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                                  const GemmParams p) {
  using namespace g2;
  constexpr int kSt = stages_for(EPI);
  constexpr bool kH = stages_h(EPI);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kSt * kABytes;
  uint8_t* sH = smem + kSt * kStageBytes;     // 1024-byte aligned: the h ring, or STORE's staging tiles
  uint8_t* bar_base = sH + side_bytes(EPI);
  uint64_t* bars = reinterpret_cast<uint64_t*>(bar_base);
  uint64_t* full = bars;                      // used in the leader
  uint64_t* empty = bars + kSt;               // both CTAs
  uint64_t* tfull = bars + 2 * kSt;           // both CTAs
  uint64_t* tempty = bars + 2 * kSt + 2;      // used in the leader
  uint64_t* drained = bars + 2 * kSt + 4;     // used in the second CTA
  uint64_t* hfull = bars + 2 * kSt + 5;       // h ring (half * kHSlots + slot): both CTAs
  uint64_t* hempty = hfull + 2 * kHSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(hempty + 2 * kHSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* row_off = reinterpret_cast<int32_t*>(bar_base + 1024);
  int32_t* tile_off = row_off + (kMaxE + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int E = p.E;
  const int NT = (EPI == EPI_SWIGLU) ? (p.N / 128) : (p.N + BN - 1) / BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2 * kHSlots; ++b) {
      mbar_init(&hfull[b], 1);
      mbar_init(&hempty[b], 4);   // the four epilogue warps of a half
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
    if (kH || (EPI == EPI_STORE && p.tma_out)) tma_prefetch_desc(&tmX);
    if (kH) tma_prefetch_desc(&tmY);
  }
  if (warp == 3) {
    int carry_r = 0, carry_t = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int n = (e < E) ? p.split_sizes[e] : 0;
      const int tiles = (e < E) ? ((n + BM - 1) / BM) * NT : 0;
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
  cluster_sync();   // both CTAs' barriers are initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  TileWalker<false, BM> walk{row_off, tile_off, E, 0, NT, p.K, nullptr};
  const int total = walk.total();
  const int num_kb = (p.K + BK - 1) / BK;   // a partial last stage reads zeros past K

  if (warp == 0) {
    // ---------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      ArmedRing ring;
      bool ok = true;
      for (int t = pair; t < total && ok && !p.stall_loads; t += npairs) {
        const TileInfo ti = walk.decode(t);
        const int a_row = ti.row0 + BMC * (int)rank;
        // this CTA's half of B: columns (MN-major) or rows (K-major) [b0, b0 + 128)
        const int b0 =
            (EPI == EPI_SWIGLU) ? (rank == 0 ? 0 : p.F) + ti.n_blk * 128 : ti.n_blk * BN + 128 * (int)rank;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          if (leader) {
            mbar_arrive_expect_tx(&full[stage], 2 * kStageBytes);
            ring.arm(stage, phase);
          }
          tma_load_4d_pair(sA + stage * kABytes, &tmA, &full[stage], 0, a_row, 2 * kb, 0);
          if (B_MN)
            tma_load_4d_pair(sB + stage * kBBytes, &tmB, &full[stage], 0, kb * BK, b0 / 64, ti.e);
          else
            tma_load_4d_pair(sB + stage * kBBytes, &tmB, &full[stage], 0, b0, 2 * kb, ti.e);
          if (++stage == kSt) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // no copy may still be landing when either CTA leaves
      pair_producer_drain(leader, ok, drained, p.timeout_ns, full, kSt, ring);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (pair leader)
    if (leader) {
      constexpr uint32_t idesc = make_idesc_bf16(BM, BN, false, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int lt = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs, ++lt) {
        const TileInfo ti = walk.decode(t);
        const int acc = lt & 1;
        if (!mbar_wait_bounded<true>(&tempty[acc], ((lt >> 1) & 1) ^ 1, abort_flag, p.timeout_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t a_addr = smem_u32(sA + stage * kABytes);
            const uint32_t b_addr = smem_u32(sB + stage * kBBytes);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              // K-major: chunk kk/4, 32 bytes per 16 k; MN-major: 16 k rows = 2048 bytes,
              // column chunks kChunkBytes apart
              const uint32_t koff = (uint32_t)(kk >> 2) * kChunkBytes + (uint32_t)(kk & 3) * 32;
              const uint64_t adesc = make_sdesc(a_addr + koff, 16, 1024, 2);
              const uint64_t bdesc = B_MN ? make_sdesc(b_addr + kk * 2048, kChunkBytes, 1024, 2)
                                          : make_sdesc(b_addr + koff, 16, 1024, 2);
              mma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit_pair(&empty[stage]);
          }
          __syncwarp();
          if (++stage == kSt) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (lane == 0) mma_commit_pair(&tfull[acc]);
        __syncwarp();
      }
    }
  } else if (kH && warp == 3) {
    // ------------------------- h loader (both CTAs; SwiGLU backward): for every tile, the
    // saved g and u of this CTA's 128 rows, one 32-column strip at a time, into each
    // half's ring in the order the half drains them (half h: strips 4h, 4h+1, ...)
    if (lane == 0) {
      ArmedRing hring;   // slots half * kHSlots + slot
      int hs[2] = {0, 0};
      uint32_t hph[2] = {0, 0};
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs) {
        const TileInfo ti = walk.decode(t);
        const int r0 = ti.row0 + BMC * (int)rank;   // past R: zero-filled; past the expert: unused
        const int n0 = ti.n_blk * BN;
        for (int it = 0; it < 4 && ok; ++it) {
          for (int hf = 0; hf < 2; ++hf) {
            const int c = 4 * hf + it;
            const int b = hf * kHSlots + hs[hf];
            if (!mbar_wait_bounded(&hempty[b], hph[hf] ^ 1, abort_flag, p.timeout_ns)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&hfull[b], kHSlotBytes);
            hring.arm(b, hph[hf]);
            uint8_t* dst = sH + b * kHSlotBytes;
            tma_load_3d(dst, &tmX, &hfull[b], n0 + 32 * c, r0, 0);
            tma_load_3d(dst + kHSlotBytes / 2, &tmX, &hfull[b], p.F + n0 + 32 * c, r0, 0);
            if (++hs[hf] == kHSlots) {
              hs[hf] = 0;
              hph[hf] ^= 1;
            }
          }
        }
      }
      // no copy may still be landing when the CTA leaves
      hring.drain(hfull, 2 * kHSlots, p.timeout_ns);
    }
  } else if (warp >= 4) {
    // -------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r_local = q * 32 + lane;
    const uint32_t tempty_leader0 = map_to_rank(smem_u32(&tempty[0]), 0);
    // SwiGLU backward: this half's position in its h ring; a thread reads its row's 64
    // bytes of g and of u (16-byte chunk j of row r at r * 64 + 16 * (j ^ ((r >> 1) & 3)))
    int hs = 0;
    uint32_t hph = 0;
    auto h_fetch = [&](uint4 (&g)[4], uint4 (&u)[4]) {
      const int b = half * kHSlots + hs;
      const bool ok = mbar_wait_bounded(&hfull[b], hph, abort_flag, p.timeout_ns);
      const uint8_t* base = sH + b * kHSlotBytes + r_local * 64;
      const int sw = (r_local >> 1) & 3;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        g[j] = *reinterpret_cast<const uint4*>(base + ((j ^ sw) << 4));
        u[j] = *reinterpret_cast<const uint4*>(base + kHSlotBytes / 2 + ((j ^ sw) << 4));
      }
      // the slot's next fill is a TMA (async-proxy) write: order these reads before it
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&hempty[b]);
      if (++hs == kHSlots) {
        hs = 0;
        hph ^= 1;
      }
      return ok;
    };
    int lt = 0;
    for (int t = pair; t < total; t += npairs, ++lt) {
      const TileInfo ti = walk.decode(t);
      const int acc = lt & 1;
      if (!mbar_wait_bounded(&tfull[acc], (lt >> 1) & 1, abort_flag, p.timeout_ns)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + acc * BN + ((uint32_t)(q * 32) << 16);
      const int w_row = BMC * (int)rank + q * 32;   // this warp's first row of the tile
      if (kH)
        bf16_epilogue_tile<EPI>(p, ti, t_row, half, BMC * (int)rank + r_local, BM, h_fetch,
                                Bf16Stager{sH + 2 * kHSlots * kHSlotBytes + (warp - 4) * kStgBytes, &tmY});
      else if (EPI == EPI_STORE && p.tma_out && w_row + 32 <= ti.rows)
        g2_store_tma(p, &tmX, sH + (warp - 4) * kStgBytes, ti, t_row, half, (long long)ti.row0 + w_row, lane);
      else
        bf16_epilogue_tile<EPI>(p, ti, t_row, half, BMC * (int)rank + r_local, BM);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + acc * 8);
    }
    // the tile stores must have completed before the CTA (and its shared memory) goes
    if ((EPI == EPI_STORE || kH) && lane == 0) bulk_wait_group0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync();   // neither CTA leaves while the other can still signal it
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace moe
