// MXFP8 grouped GEMM on a pair of SMs (tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale),
// M-grouped (ragged expert rows): fc1 + ScaledSwiGLU + MXFP8 quantisation, fc2, and the
// two data-gradient GEMMs of the backward.
//
// Pages: "Efficient MoE training for biological foundation models" (news.bpdata.com
// sections 2-3: MXFP8 operands with one scale per 32 K values consumed by the tensor
// cores, the fused GroupedLinear -> ScaledSwiGLU -> GroupedLinear chain).
//
// A 2-CTA cluster computes 256 x 256 output tiles; the pair leader issues M=256, N=256,
// K=32 MMAs that read each CTA's 128 rows of A and 128 rows (its half) of B.
//
// Feeding: issuing a TMA copy costs about the same whatever its size, so a copy per
// 512-byte scale atom every 128-wide k-block starved the tensor pipe. Here
//   * a k-stage is 256 wide: ONE copy per operand per stage brings two 128-byte k-chunks
//     of 128 rows (a 4-D view of the codes, box {128, 128, 2, 1}): 64 KB per CTA, 3 stages;
//   * scale atoms travel on their own two-slot ring, four k-blocks per copy (2 KB): per
//     two stages, one copy for this CTA's A rows and two for the B tile's two 128-row
//     groups (the block-scaled pair MMA reads every N column's scales from each CTA's own
//     tensor memory, so both CTAs fetch both B groups). Warp 2 of the leader copies each
//     k-block's atoms into both CTAs' tensor memory (tcgen05.cp.cta_group::2), into the
//     next of four scale sets, ahead of the MMA thread (ScaleCopier).
//
// The SwiGLU backward's epilogue also needs the saved h = [g | u] of every row it drains:
// warp 3 of each CTA copies it with TMA into a shared-memory ring of 32-column strips,
// ahead of the epilogue, which reads its row from there (coalesced copies instead of one
// 16-byte load per row and lane from global memory).
//
// Its dh code tiles (32 rows x 32 codes, in both quantised forms) leave through a 1 KB
// shared-memory staging tile per epilogue warp with one TMA store each, for warps whose
// rows all belong to the tile's expert.
//
// Tensor memory per CTA: overlapping accumulators acc0 = [0, 256) and acc1 = [192, 448),
// four scale sets at 448..495; `tovl` and `tempty` live in the leader and count
// one arrival per epilogue warp of both CTAs. Waits are bounded like in every other
// kernel of this library.
#pragma once
#include "grouped_gemm_mxf8_sm100.cuh"

namespace moe {

namespace mx2 {
constexpr int BM = 256;                       // rows of a pair tile
constexpr int BMC = 128;                      // rows per CTA
constexpr int BN = 256;
#ifndef MOE_MX2_CHUNKS
#define MOE_MX2_CHUNKS 2
#endif
#ifndef MOE_MX2_STAGES
#define MOE_MX2_STAGES 3
#endif
constexpr int kChunks = MOE_MX2_CHUNKS;       // 128-byte k-chunks per stage (1 or 2)
constexpr int BK = 128 * kChunks;             // k per stage
constexpr int kStages = MOE_MX2_STAGES;
constexpr int kThreads = 384;
constexpr int kChunkBytes = 128 * 128;        // one k-chunk of 128 rows, 16 KB
constexpr int kABytes = BMC * BK;             // 16 KB per chunk
constexpr int kBBytes = (BN / 2) * BK;        // 16 KB per chunk: this CTA's half of B
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kSfKb = 4;                      // k-blocks (of 128) per scale copy
constexpr int kSfGroupBytes = kSfKb * 512;    // 2 KB: one row group's atoms for kSfKb k-blocks
constexpr int kSfSlotBytes = 3 * kSfGroupBytes;   // A group, B lower group, B upper group
constexpr int kSfSlots = 2;
constexpr int kStPerSf = kSfKb / kChunks;     // stages per scale slot
static_assert(kChunks == 1 || kChunks == 2, "one or two k-chunks per stage");

constexpr int kMaxE = 1024;
constexpr int kTmemCols = 512;
// SwiGLU backward: the saved h reaches the epilogue through shared memory, a ring of
// 32-column strips (g and u of the CTA's 128 rows, 64-byte swizzled: 16 KB) per column
// half; its 64 KB come out of the operand ring, which keeps the stages that remain (the
// K = H mainloop of that GEMM is shorter than its epilogue).
constexpr int kHSlotBytes = 2 * 128 * 64;
constexpr int kHSlots = 2;                    // per half
__host__ __device__ constexpr bool stages_h(int epi) { return epi == MXEPI_DSWIGLU; }
__host__ __device__ constexpr int stages_for(int epi) {
  return stages_h(epi) ? kStages - (2 * kHSlots * kHSlotBytes + kStageBytes - 1) / kStageBytes : kStages;
}
// SwiGLU backward: a 1 KB staging tile (32 rows x 32 codes) per epilogue warp for the TMA
// stores of dh's code tiles
constexpr int kCodeStgBytes = 32 * 32;
__host__ __device__ constexpr int side_bytes(int epi) {
  return stages_h(epi) ? 2 * kHSlots * kHSlotBytes + 8 * kCodeStgBytes : 0;
}
__host__ __device__ constexpr int smem_bytes(int epi) {
  return 1024 + stages_for(epi) * kStageBytes + kSfSlots * kSfSlotBytes + side_bytes(epi) + 1024 +
         3 * (kMaxE + 1) * 4;
}
static_assert(smem_bytes(MXEPI_DSWIGLU) <= 232448 && smem_bytes(MXEPI_STORE) <= 232448, "shared memory per CTA");
}  // namespace mx2

// tmA / tmB: E4M3 codes [rows, K] / [E][b_rows][K] as {128, rows, K/128 chunks, batch},
// box {128, 128, 2, 1}. tmSa / tmSb: scale atoms as uint32 tensors {128 words, K/128
// k-blocks, row groups} with a box of four atoms (no swizzle); A's row groups are the
// experts' 128-row tiles in order, B's are e * (b_rows / 128) + row / 128.
// tmH (SwiGLU backward only): the saved h [R, 2F] bf16 as {2F, R, 1}, box {32, 128},
// 64-byte swizzle; tmDc / tmDr (SwiGLU backward only): dh_cols / dh_rows codes [R, 2F] as
// {2F, R, 1}, box {32, 32}, 32-byte swizzle.
template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(mx2::kThreads, 1)
    grouped_gemm_mxf8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                  const __grid_constant__ CUtensorMap tmSa, const __grid_constant__ CUtensorMap tmSb,
                                  const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmDc,
                                  const __grid_constant__ CUtensorMap tmDr, const MxGemmParams mp) {
  using namespace mx2;
  constexpr int kSt = stages_for(EPI);
  constexpr bool kH = stages_h(EPI);
  // ScaleCopier waits for the `empty` phase of the stage kSfSets k-blocks back; the MMA
  // thread can complete at most kSfSets / kChunks - 1 later stages meanwhile, which must
  // stay below the ring's kSt (else that slot's barrier could be two phases ahead)
  static_assert(mx::kSfSets <= kSt * kChunks, "operand ring too short for the scale-set look-back");
  const GemmParams& p = mp.g;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kSt * kABytes;
  uint8_t* sSf = sB + kSt * kBBytes;
  uint8_t* sH = sSf + kSfSlots * kSfSlotBytes;  // 1024-byte aligned: kSfSlots * kSfSlotBytes = 12 KB
  uint8_t* sStg = sH + (kH ? 2 * kHSlots * kHSlotBytes : 0);   // SwiGLU backward: code staging tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sH + side_bytes(EPI));
  uint64_t* full = bars;                      // used in the leader
  uint64_t* empty = bars + kSt;               // both CTAs
  uint64_t* tfull = bars + 2 * kSt;           // both CTAs
  uint64_t* tempty = bars + 2 * kSt + 2;      // used in the leader
  uint64_t* tovl = bars + 2 * kSt + 4;        // used in the leader
  uint64_t* sfull = bars + 2 * kSt + 5;       // scale ring: used in the leader
  uint64_t* sempty = sfull + kSfSlots;        // scale ring: both CTAs
  uint64_t* drained = sempty + kSfSlots;      // used in the second CTA
  uint64_t* hfull = drained + 1;              // h ring (half * kHSlots + slot): both CTAs
  uint64_t* hempty = hfull + 2 * kHSlots;
  uint64_t* setfull = hempty + 2 * kHSlots;   // tensor-memory scale sets: used in the leader
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(setfull + mx::kSfSets);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* row_off = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(bars) + 1024);
  int32_t* tile_off = row_off + (kMaxE + 1);
  int32_t* grp_off = tile_off + (kMaxE + 1);  // 128-row scale groups of earlier experts

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int E = p.E;
  const int NT = mx_swiglu(EPI) ? (p.N / 128) : (p.N + BN - 1) / BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2 * kHSlots; ++b) {
      mbar_init(&hfull[b], 1);
      mbar_init(&hempty[b], 4);   // the four epilogue warps of a half
    }
    for (int b = 0; b < mx::kSfSets; ++b) {
      mbar_init(&setfull[b], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 16);   // 8 epilogue warps in each CTA of the pair
    }
    mbar_init(tovl, 16);
    for (int s2 = 0; s2 < kSfSlots; ++s2) {
      mbar_init(&sfull[s2], 1);
      mbar_init(&sempty[s2], 1);
    }
    mbar_init(drained, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSa);
    tma_prefetch_desc(&tmSb);
    if (kH) {
      tma_prefetch_desc(&tmH);
      tma_prefetch_desc(&tmDc);
      tma_prefetch_desc(&tmDr);
    }
  }
  if (warp == 3) {
    int carry_r = 0, carry_t = 0, carry_g = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int n = (e < E) ? p.split_sizes[e] : 0;
      const int tiles = (e < E) ? ((n + BM - 1) / BM) * NT : 0;
      const int grps = (n + BMC - 1) / BMC;
      int ir = n, it = tiles, ig = grps;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yr = __shfl_up_sync(0xffffffffu, ir, o);
        const int yt = __shfl_up_sync(0xffffffffu, it, o);
        const int yg = __shfl_up_sync(0xffffffffu, ig, o);
        if (lane >= o) {
          ir += yr;
          it += yt;
          ig += yg;
        }
      }
      if (e < E) {
        row_off[e] = carry_r + ir - n;
        tile_off[e] = carry_t + it - tiles;
        grp_off[e] = carry_g + ig - grps;
      }
      carry_r += __shfl_sync(0xffffffffu, ir, 31);
      carry_t += __shfl_sync(0xffffffffu, it, 31);
      carry_g += __shfl_sync(0xffffffffu, ig, 31);
    }
    if (lane == 0) {
      row_off[E] = carry_r;
      tile_off[E] = carry_t;
      grp_off[E] = carry_g;
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
  const int kblocks = p.K / 128;                      // 128-wide k-blocks (K is a multiple of 128)
  const int num_st = (kblocks + kChunks - 1) / kChunks;   // stages; a partial last stage reads zeros past K

  if (warp == 0) {
    // ---------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0, sslot = 0;
      uint32_t phase = 0, sphase = 0;
      ArmedRing ring, sring;
      bool ok = true;
      const int bgroups = mp.b_rows / 128;
      for (int t = pair; t < total && ok && !p.stall_loads; t += npairs) {
        const TileInfo ti = walk.decode(t);
        const int n0 = mx_swiglu(EPI) ? ti.n_blk * 128 : ti.n_blk * BN;
        // this CTA's A rows and their scale group (past the expert: unused rows; a group
        // index past the atom tensor reads zeros)
        const int a_row = ti.row0 + BMC * (int)rank;
        const int ga = grp_off[ti.e] + 2 * ti.m_blk + (int)rank;
        // this CTA's half of B, and the scale groups of both halves
        const int b_row = mx_swiglu(EPI) ? (rank ? p.F : 0) + n0 : n0 + 128 * (int)rank;
        const int gb0 = ti.e * bgroups + n0 / 128;
        int gb1 = mx_swiglu(EPI) ? ti.e * bgroups + (p.F + n0) / 128 : gb0 + 1;
        if (!mx_swiglu(EPI) && n0 + 128 >= mp.b_rows) gb1 = gb0;   // past N: codes are zero-filled
        for (int st = 0; st < num_st; ++st) {
          if (st % kStPerSf == 0) {
            // scale atoms of k-blocks [kChunks st, kChunks st + 4) (past K: zeros)
            if (!mbar_wait_bounded(&sempty[sslot], sphase ^ 1, abort_flag, p.timeout_ns)) {
              ok = false;
              break;
            }
            if (leader) {
              mbar_arrive_expect_tx(&sfull[sslot], 2 * kSfSlotBytes);
              sring.arm(sslot, sphase);
            }
            uint8_t* sd = sSf + sslot * kSfSlotBytes;
            tma_load_3d_pair(sd, &tmSa, &sfull[sslot], 0, kChunks * st, ga);
            tma_load_3d_pair(sd + kSfGroupBytes, &tmSb, &sfull[sslot], 0, kChunks * st, gb0);
            tma_load_3d_pair(sd + 2 * kSfGroupBytes, &tmSb, &sfull[sslot], 0, kChunks * st, gb1);
            if (++sslot == kSfSlots) {
              sslot = 0;
              sphase ^= 1;
            }
          }
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          if (leader) {
            mbar_arrive_expect_tx(&full[stage], 2 * kStageBytes);
            ring.arm(stage, phase);
          }
          tma_load_4d_pair(sA + stage * kABytes, &tmA, &full[stage], 0, a_row, kChunks * st, 0);
          tma_load_4d_pair(sB + stage * kBBytes, &tmB, &full[stage], 0, b_row, kChunks * st, ti.e);

          if (++stage == kSt) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // no copy may still be landing when either CTA leaves
      pair_producer_drain(leader, ok, drained, p.timeout_ns, full, kSt, ring, sfull, kSfSlots, &sring);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (pair leader)
    if (leader) {
      int stage = 0;
      uint32_t phase = 0;
      int lt = 0;
      bool ok = true;
      ScaleSets sets{setfull, tmem_base};
      for (int t = pair; t < total && ok; t += npairs, ++lt) {
        const int acc = lt & 1;
        if (!mbar_wait_bounded<true>(&tempty[acc], ((lt >> 1) & 1) ^ 1, abort_flag, p.timeout_ns)) break;
        if (lt > 0 && !mbar_wait_bounded<true>(tovl, (lt - 1) & 1, abort_flag, p.timeout_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (acc ? mx::kAcc1Col : 0u);
        for (int st = 0; st < num_st && ok; ++st) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          const uint32_t a_addr = smem_u32(sA + stage * kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * kBBytes);
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            const int kb = kChunks * st + c;
            if (kb >= kblocks) break;
            // this k-block's scale atoms, copied into tensor memory by the scale warp
            if (!sets.wait(abort_flag, p.timeout_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (lane == 0) {
              const uint32_t sfa = sets.sfa(), sfb = sets.sfb();
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t adesc = make_sdesc(a_addr + c * kChunkBytes + kk * 32, 16, 1024, 2);
                const uint64_t bdesc = make_sdesc(b_addr + c * kChunkBytes + kk * 32, 16, 1024, 2);
                const uint32_t idesc = make_idesc_mxf8(BM, BN, false, false, kk, kk) | mp.ab_fmt;
                mma_mxf8_pair(d_tmem, adesc, bdesc, idesc, sfa | ((uint32_t)kk << 30), sfb | ((uint32_t)kk << 30),
                              (kb > 0 || kk > 0) ? 1u : 0u);
              }
            }
            sets.next();
            __syncwarp();
          }
          if (!ok) break;
          if (lane == 0) mma_commit_pair(&empty[stage]);
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
  } else if (warp == 2) {
    // ------------------------------------ scale copies (pair leader): every k-block's
    // atoms into the next tensor-memory scale set, ahead of the MMA thread
    if (leader && lane == 0) {
      ScaleCopier<kSfKb> cp{sfull, sempty, setfull, empty, kSt, sSf, kSfSlots, tmem_base, abort_flag, p.timeout_ns};
      bool ok = true;
      int g0 = 0;   // global stage of the tile's first k-block
      for (int t = pair; t < total && ok; t += npairs, g0 += num_st)
        for (int kb = 0; kb < kblocks && ok; ++kb) ok = cp.copy(kb, kb == kblocks - 1, g0 + kb / kChunks);
      cp.drain();
    }
  } else if (kH && warp == 3) {
    // ------------------------- h loader (both CTAs; SwiGLU backward): for every tile, the
    // saved g and u of this CTA's 128 rows, one 32-column strip at a time, into each
    // half's ring in the order that half's epilogue warps drain the strips
    if (lane == 0) {
      ArmedRing hring;   // slots half * kHSlots + slot
      int hs[2] = {0, 0};
      uint32_t hph[2] = {0, 0};
      bool ok = true;
      int lt = 0;
      for (int t = pair; t < total && ok; t += npairs, ++lt) {
        const TileInfo ti = walk.decode(t);
        const int acc = lt & 1;
        const int r0 = ti.row0 + BMC * (int)rank;   // past R: zero-filled; past the expert: unused
        const int n0 = ti.n_blk * BN;
        for (int it = 0; it < 4 && ok; ++it) {
          for (int hf = 0; hf < 2; ++hf) {
            const int c = strip8(acc, hf, it);
            const int b = hf * kHSlots + hs[hf];
            if (!mbar_wait_bounded(&hempty[b], hph[hf] ^ 1, abort_flag, p.timeout_ns)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&hfull[b], kHSlotBytes);
            hring.arm(b, hph[hf]);
            uint8_t* dst = sH + b * kHSlotBytes;
            tma_load_3d(dst, &tmH, &hfull[b], n0 + 32 * c, r0, 0);
            tma_load_3d(dst + kHSlotBytes / 2, &tmH, &hfull[b], p.F + n0 + 32 * c, r0, 0);
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
    const uint32_t tovl_leader = map_to_rank(smem_u32(tovl), 0);
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
      // the slot's next fill is a TMA (async-proxy) write: order these generic-proxy reads
      // before it, or the copy can land under reads still in flight (seen as
      // run-to-run differences in a few strips without this fence)
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
      const uint32_t t_row = tmem_base + (acc ? mx::kAcc1Col : 0u) + ((uint32_t)(q * 32) << 16);
      const uint32_t sc_word = mxf8_epilogue_tile<EPI>(
          mp, ti, t_row, acc, half, BMC * (int)rank + r_local, BM,
          [&] {
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tovl_leader);
          },
          grp_off[ti.e], row_off[ti.e + 1] - row_off[ti.e], h_fetch,
          kH ? CodeStager{sStg + (warp - 4) * kCodeStgBytes, &tmDc, &tmDr} : CodeStager{});
      if (EPI == MXEPI_SWIGLU_Q && BMC * (int)rank < ti.rows) {
        // this CTA's 128 rows form scale group grp_off[e] + 2 m_blk + rank of `a`: the bytes
        // of this half's two a-strips (rows past the expert store 0; a CTA entirely past
        // the expert writes nothing)
        const size_t g = (size_t)(grp_off[ti.e] + 2 * ti.m_blk + (int)rank);
#pragma unroll
        for (int it = 0; it < 2; ++it) {
          const int c = strip4(acc, half, it);
          mp.out_atoms[mma_scale_offset(g, r_local, 4 * ti.n_blk + c, p.N / 128)] = (uint8_t)(sc_word >> (8 * c));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + acc * 8);
    }
    // the code tiles' stores must have completed before the CTA (and its shared memory) goes
    if (kH && lane == 0) bulk_wait_group0();
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
