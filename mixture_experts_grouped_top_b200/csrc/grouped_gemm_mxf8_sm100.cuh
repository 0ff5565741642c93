// MXFP8 pieces shared by the block-scaled grouped GEMMs on sm_100a: E4M3 (or E5M2) A and
// B with one E8M0 scale per 32 consecutive K values, fp32 accumulation in tensor memory
// (tcgen05.mma kind::mxf8f6f4.block_scale, K=32 per instruction): the parameter block, the
// warp-level quantisers and the fused epilogues that drain a 128-row x 256-column
// accumulator.
//
// Pages: "Efficient MoE training for biological foundation models" (news.bpdata.com
// section 2: MXFP8 keeps one scale per block of 32 consecutive values and Blackwell
// tensor cores consume it directly; section 3: the fused GroupedLinear -> ScaledSwiGLU ->
// GroupedLinear chain with quantisation fused into it).
//
// The kernels live in grouped_gemm_mxf8_pair_sm100.cuh (M-grouped: fc1, fc2 and the two
// data gradients) and grouped_gemm_mxf8_kgroup_pair_sm100.cuh (K-grouped weight
// gradients), both on CTA pairs. What is specific to block scaling:
//   * scales are 512-byte atoms per 128-wide k-block (128 rows x 4 scale bytes, row r of
//     the group at word (r % 32) * 4 + r / 32, the layout tcgen05.cp expects), already
//     arranged so in global memory (mma_scale_offset), a row group's atoms for
//     consecutive k-blocks contiguous: they travel on a two-slot ring of their own, one
//     copy per row group (A, and B's two 128-row halves) per four k-blocks, since a copy
//     costs the copy engine about the same whatever its size;
//   * a warp of its own moves each k-block's atoms into tensor memory with tcgen05.cp
//     (32 lanes x 16 B, replicated to the four sub-partitions), into the next of four
//     scale sets, ahead of the MMA thread, which issues the four K=32 MMAs of the k-block
//     from that set, selecting scale byte kk of each word through the scale-factor ids.
//     Copies issued by the MMA thread itself, right before its MMAs, held its tensor-core
//     stream (tensor pipe active 65% with them, 82% with the copies on another warp: fc2 of
//     the Mixtral MXFP8 forward, 2048 tokens), and with only two sets the handoff between
//     the warps left the MMA thread waiting (56%); see ScaleCopier;
//   * two 256-column accumulators plus the scale sets exceed the 512 tensor-memory
//     columns, so the accumulators overlap: acc0 = columns [0, 256), acc1 = [192, 448),
//     four 12-column scale sets at [448, 496). The epilogue drains the two shared 32-column
//     strips first (one per half, strip8 / strip4) and signals `tovl`; the next tile's MMAs
//     wait for them (and for the full drain of the tile two back) instead of the whole
//     previous epilogue.
#pragma once
#include "grouped_gemm_sm100.cuh"
#include "token_kernels.cuh"

namespace moe {

namespace mx {
// tensor-memory layout shared by the MXFP8 pair kernels (columns of each CTA's 512)
constexpr int BN = 256;                       // accumulator columns per tile
constexpr uint32_t kAcc1Col = 192;            // acc0 = [0, 256), acc1 = [192, 448)
constexpr uint32_t kSfaCol = 448;             // A scales of set 0: 4 columns
constexpr uint32_t kSfbCol = 452;             // B scales of set 0: 2 x 4 columns
constexpr uint32_t kSfSetCols = 12;           // set s at 448 + 12 s
constexpr int kSfSets = 4;                    // [448, 496)
}  // namespace mx

enum MxEpiKind : int {
  MXEPI_STORE = 0,      // out[row, col] = bf16(acc) (fp32 with out_f32)
  MXEPI_SWIGLU_Q = 1,   // a = SiLU(g) * u * p quantised to MXFP8 along the columns (+ bf16 h)
  MXEPI_DSWIGLU = 2,    // SwiGLU backward from da = acc and the saved h: dh (MXFP8, both axes), dprob partials
  MXEPI_WGRAD = 3,      // K-grouped: out[e, m, n] = bf16(acc), zeros for an expert without rows
  MXEPI_SWIGLU_F8 = 4,  // per-tensor FP8 fc1: a = SiLU(g) * u * p stored bf16 (+ bf16 h), max |a| kept
  MXEPI_DSWIGLU_F8 = 5, // per-tensor FP8 fc2 dgrad: dh stored bf16, max |dh| kept, dprob partials
};

// fc1 epilogues (N tiles pair gate columns with their up columns)
__host__ __device__ constexpr bool mx_swiglu(int epi) { return epi == MXEPI_SWIGLU_Q || epi == MXEPI_SWIGLU_F8; }

struct MxGemmParams {
  GemmParams g;               // E, M (rows R), N (output cols), K, split_sizes, out, ldo, out2/ldo2 (h), probs, F
  // M-grouped: A scale atoms grouped per expert tile (sum of ceil(n_e/128)), B scale atoms
  // grouped e * (b_rows / 128) + row / 128. K-grouped (MN-major codes [R, M] and [R, N]):
  // atoms per expert, k-group and column group, as quant_cols_grouped_kernel writes them.
  const uint8_t* a_atoms;
  const uint8_t* b_atoms;
  int b_rows;                 // rows of each expert's B (2F for fc1, H for fc2)
  uint8_t* out_atoms;         // MXEPI_SWIGLU_Q: scales of `a` as atoms for the next GEMM (K = F)
  // MXEPI_DSWIGLU: the MXFP8 operands of the backward's remaining GEMMs, quantised in the
  // epilogue: dh = [dg | du] along its columns (codes [R, 2F], tile atoms, K = 2F) and
  // along each expert's rows (codes [R, 2F], grouped atoms).
  // MXEPI_SWIGLU_Q in training: a along each expert's rows (codes [R, F], grouped atoms)
  // for the fc2 weight gradient.
  uint8_t* dh_rows;
  uint8_t* dh_rows_atoms;
  uint8_t* dh_cols;
  uint8_t* dh_cols_atoms;
  uint8_t* a_cols;
  uint8_t* a_cols_atoms;
  // Per-tensor FP8 (the operands are E4M3 / E5M2 codes with one scale per tensor; their
  // block scales are all 2^0): ab_fmt is OR-ed into every instruction descriptor (A's
  // format at bit 7, B's at bit 10: 0 = E4M3, 1 = E5M2); with deq_a set, the epilogue
  // multiplies the accumulator by 1 / (deq_a[0] * deq_b[e]) (M-grouped: B's scale per
  // expert; K-grouped: deq_b[0]); amax_out collects max |x| of the bf16 output (fp32 bits).
  uint32_t ab_fmt;
  const float* deq_a;
  const float* deq_b;
  unsigned int* amax_out;
};

// 1 / (s_a s_b) of a per-tensor FP8 GEMM, 1 otherwise.
__device__ __forceinline__ float mx_deq_factor(const MxGemmParams& mp, int e) {
  return mp.deq_a ? 1.0f / (mp.deq_a[0] * mp.deq_b[e]) : 1.0f;
}

// max over the warp of a non-negative float, folded into *out (fp32 bits, atomicMax):
// every lane of the warp must call this together.
__device__ __forceinline__ void warp_amax_to(unsigned int* out, float v) {
  const unsigned int m = __reduce_max_sync(0xffffffffu, __float_as_uint(v));
  if ((threadIdx.x & 31) == 0 && m) atomicMax(out, m);
}

// Scale-set handoff between the scale-copy warp and the MMA thread of a CTA pair (both in
// the leader). The copier takes k-block kb's atoms from the scale ring in shared memory
// (slots of kPerSlot k-blocks, 3 groups of kPerSlot atoms: A, B lower, B upper) into the
// next of mx::kSfSets tensor-memory sets, round robin, and commits `setfull[set]`; the
// MMA thread waits for it and issues the k-block's MMAs from that set. A set is free again
// once the MMAs of the k-block that used it before are done: the copier learns that from
// the operand ring's `empty` barrier of that k-block's stage, which the MMA thread commits
// anyway (an extra commit per k-block held the MMA thread's stream, like the copies
// themselves). That phase is the last one the stage's slot completed as long as the
// MMA thread cannot finish another kSt stages first: kernels assert kSfSets <= kSt *
// (k-blocks per stage). The copier releases a scale-ring slot (`sempty`) once the copies
// of its last k-block are done. Bounded waits; all barriers count one arrival.
template <int kPerSlot>
struct ScaleCopier {
  uint64_t* sfull;
  uint64_t* sempty;
  uint64_t* setfull;
  uint64_t* empty;            // the operand ring's stage barriers (nstages slots)
  int nstages;
  const uint8_t* ring;        // slot s at ring + s * 3 * kPerSlot * 512
  int nslots;
  uint32_t tmem_base;
  volatile int* abort;
  uint64_t timeout_ns;
  int slot = 0, set = 0;
  uint32_t sphase = 0;
  uint32_t par = 0;           // bit s: parity of the copies committed into set s so far
  uint32_t used = 0;          // bit s: set s received copies
  int q0 = -1, q1 = -1, q2 = -1, q3 = -1;   // global stages of the last four k-blocks copied

  // the atoms of k-block kb of the current tile, whose operands are global stage `gstage`
  // of the operand ring; `last`: the tile's last k-block
  __device__ __forceinline__ bool copy(int kb, bool last, int gstage) {
    static_assert(mx::kSfSets == 4, "the stage history below holds four k-blocks");
    const int q = kb % kPerSlot;
    if (q == 0 && !mbar_wait_bounded(&sfull[slot], sphase, abort, timeout_ns)) return false;
    // the set's previous k-block (four copies back): its stage's MMAs must be done
    if (q0 >= 0 && !mbar_wait_bounded(&empty[q0 % nstages], (uint32_t)(q0 / nstages) & 1u, abort, timeout_ns))
      return false;
    q0 = q1;
    q1 = q2;
    q2 = q3;
    q3 = gstage;
    tc_fence_after();
    const uint32_t src = smem_u32(ring + (size_t)slot * 3 * kPerSlot * 512) + (uint32_t)q * 512;
    const uint32_t sfa = tmem_base + mx::kSfaCol + (uint32_t)set * mx::kSfSetCols;
    const uint32_t sfb = tmem_base + mx::kSfbCol + (uint32_t)set * mx::kSfSetCols;
    tmem_cp_32x128b_warpx4_pair(sfa, make_sdesc(src, 0, 128, 0));
    tmem_cp_32x128b_warpx4_pair(sfb, make_sdesc(src + kPerSlot * 512, 0, 128, 0));
    tmem_cp_32x128b_warpx4_pair(sfb + 4, make_sdesc(src + 2 * kPerSlot * 512, 0, 128, 0));
    mma_commit_pair(&setfull[set]);
    if (q == kPerSlot - 1 || last) {
      mma_commit_pair(&sempty[slot]);
      if (++slot == nslots) {
        slot = 0;
        sphase ^= 1u;
      }
    }
    par ^= 1u << set;
    used |= 1u << set;
    set = (set + 1) % mx::kSfSets;
    return true;
  }
  // on the way out: wait (bounded) until the last copies into each set have landed (the
  // last commit into set s completed phase parity ((par >> s) & 1) ^ 1)
  __device__ __forceinline__ void drain() const {
    for (int s_ = 0; s_ < mx::kSfSets; ++s_)
      if ((used >> s_) & 1u) mbar_wait_drain(&setfull[s_], ((par >> s_) & 1u) ^ 1u, timeout_ns);
  }
};

// The MMA thread's side of the handoff: which set the next k-block reads.
struct ScaleSets {
  uint64_t* setfull;
  uint32_t tmem_base;
  int set = 0;
  uint32_t par = 0;           // bit s: parity of the next fill of set s to wait for
  __device__ __forceinline__ bool wait(volatile int* abort, uint64_t timeout_ns) const {
    return mbar_wait_bounded(&setfull[set], (par >> set) & 1u, abort, timeout_ns);
  }
  __device__ __forceinline__ uint32_t sfa() const { return tmem_base + mx::kSfaCol + (uint32_t)set * mx::kSfSetCols; }
  __device__ __forceinline__ uint32_t sfb() const { return tmem_base + mx::kSfbCol + (uint32_t)set * mx::kSfSetCols; }
  // after the k-block's MMAs are issued (every lane advances)
  __device__ __forceinline__ void next() {
    par ^= 1u << set;
    set = (set + 1) % mx::kSfSets;
  }
};

// The 32-column strips of a 256-column accumulator that the two halves of the epilogue
// warps drain, in order: half h takes strips h, h+2, h+4, h+6 (SwiGLU epilogues: a-strips
// h and h+2, a-strip c reading gate strip c and up strip 4 + c). acc0 and acc1 share 64
// columns, acc0's strips 6 and 7 and acc1's strips 0 and 1, one per half: each half
// drains its shared strip first, so that the next tile's MMAs may start writing there.
__host__ __device__ constexpr int strip8(int acc, int half, int it) {
  return acc ? half + 2 * it : (it == 0 ? 6 + half : half + 2 * (it - 1));
}
__host__ __device__ constexpr int strip4(int acc, int half, int it) {
  return acc ? half + 2 * it : (it == 0 ? 2 + half : half);
}

// Drains one 128-row x 256-column accumulator (this thread's row: lane quadrant of
// `t_row`, row r_local of the output tile) and runs the epilogue EPI on it, strip by strip
// (strip8 / strip4); after its first strip every warp calls `strip_done()` (warp-uniform
// calls, so the callee may signal once per warp). Returns the SwiGLU_Q row's scale bytes
// (byte c: a-strip c; the bytes of the other half's strips are 0).
// DSWIGLU also takes the expert's first 128-row group (grp0: groups of earlier experts),
// its row count n_e, which place its scale atoms, and `h_fetch(g, u)`, which hands this
// thread the saved h of its row for the next 32-column strip in the order the strips are
// drained (the caller stages h in shared memory ahead of the epilogue).
// MXEPI_DSWIGLU: where a warp's dh code tiles go by TMA (null stg: lane stores). stg: the
// warp's 1 KB staging tile; tm_cols / tm_rows: dh_cols / dh_rows [R, 2F] as {2F, R, 1},
// boxes {32, 32}, 32-byte swizzle.
struct CodeStager {
  uint8_t* stg = nullptr;
  const CUtensorMap* tm_cols = nullptr;
  const CUtensorMap* tm_rows = nullptr;
};

// A warp's 32 rows x 32 E4M3 codes (w: this lane's row, starting at global row y) to
// column x of a code array by one TMA store through the warp's staging tile (32-byte
// swizzle: 16-byte chunk j of row r at r*32 + 16*(j ^ ((r>>2)&1)), conflict-free for
// these writes); lane 0 first waits until the tile's previous store has read it. Lane
// stores of 32 bytes per row made 32 separate L2 requests per instruction, about a
// fifth of the SwiGLU backward's time at the genomic size.
__device__ __forceinline__ void store_codes_tma(uint8_t* stg, const CUtensorMap* tm, int x, int y,
                                                const uint32_t (&w)[8], int lane) {
  if (lane == 0) bulk_wait_group_read0();
  __syncwarp();
  uint8_t* row = stg + lane * 32;
  const int sw = (lane >> 2) & 1;
  *reinterpret_cast<uint4*>(row + 16 * sw) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(row + 16 * (sw ^ 1)) = make_uint4(w[4], w[5], w[6], w[7]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_3d(tm, stg, x, y, 0);
    bulk_commit_group();
  }
}

template <int EPI, class StripDone, class HFetch = NoHFetch>
__device__ __forceinline__ uint32_t mxf8_epilogue_tile(const MxGemmParams& mp, const TileInfo& ti, uint32_t t_row,
                                                       int acc, int half, int r_local, int tile_bm,
                                                       StripDone&& strip_done, int grp0 = 0, int n_e = 0,
                                                       const HFetch& h_fetch = HFetch{},
                                                       const CodeStager& cs = CodeStager{}) {
  using mx::BN;
  const GemmParams& p = mp.g;
  const bool row_ok = r_local < ti.rows;
  const long long row = ti.row0 + r_local;
  uint32_t sc_word = 0;   // SwiGLU: this row's four scale bytes (k-blocks 4*n_blk..+3 of the next GEMM)

  if (EPI == MXEPI_STORE || EPI == MXEPI_WGRAD) {
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
    const int n0 = ti.n_blk * BN;
    long long orow;
    bool ok_row;
    bool zero = false;
    if (EPI == MXEPI_WGRAD) {
      const int m = ti.m_blk * tile_bm + r_local;
      ok_row = m < p.M;
      orow = (long long)ti.e * p.out_batch + (long long)m * p.ldo;
      zero = ti.rows == 0;
    } else {
      ok_row = row_ok;
      orow = row * p.ldo;
    }
    const float deq = mx_deq_factor(mp, EPI == MXEPI_WGRAD ? 0 : ti.e);
#pragma unroll 1
    for (int it = 0; it < 4; ++it) {
      const int c = strip8(acc, half, it);
      uint32_t v0[16], v1[16];
      tmem_ld_32x32b_x16(t_row + c * 32, v0);
      tmem_ld_32x32b_x16(t_row + c * 32 + 16, v1);
      tmem_wait_ld();
      if (it == 0) {
        tc_fence_before();
        strip_done();
      }
      if (mp.deq_a) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          v0[i] = __float_as_uint(__uint_as_float(v0[i]) * deq);
          v1[i] = __float_as_uint(__uint_as_float(v1[i]) * deq);
        }
      }
      if (EPI == MXEPI_STORE && ok_row && n0 + c * 32 < p.N && p.row_token) {
        float* d = p.out32 + (long long)p.row_token[row] * p.ldo + n0 + c * 32;
        combine_add16(d, v0);
        combine_add16(d + 16, v1);
      } else if (ok_row && n0 + c * 32 < p.N && p.out_f32) {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<float*>(p.out) + orow + n0 + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          dst[i] = make_uint4(v0[4 * i], v0[4 * i + 1], v0[4 * i + 2], v0[4 * i + 3]);
          dst[4 + i] = make_uint4(v1[4 * i], v1[4 * i + 1], v1[4 * i + 2], v1[4 * i + 3]);
        }
      } else if (ok_row && n0 + c * 32 < p.N) {
        uint4 o[4];
        uint32_t* ow = reinterpret_cast<uint32_t*>(o);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          ow[i] = zero ? 0u : pack_bf16x2(__uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1]));
          ow[8 + i] = zero ? 0u : pack_bf16x2(__uint_as_float(v1[2 * i]), __uint_as_float(v1[2 * i + 1]));
        }
        uint4* dst = reinterpret_cast<uint4*>(out + orow + n0 + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = o[i];
      }
    }
  } else if (EPI == MXEPI_DSWIGLU) {
    // acc = da for columns [n0, n0+256) of F. With h = [g | u] from the forward:
    // dg = da p u SiLU'(g), du = da p SiLU(g), dp += da SiLU(g) u. dh = [dg | du] is
    // quantised here from fp32 into the operands of the GEMMs that follow (see
    // MxGemmParams): along its columns (this row's 32-column blocks) and along the
    // expert's rows (32-row blocks = this warp's lanes: a pair tile starts at a multiple
    // of 256 rows of its expert, so the blocks restart at every expert; lanes past the
    // expert's end count as zeros).
    const float pr = (row_ok && p.probs) ? p.probs[row] : 1.0f;
    const int n0 = ti.n_blk * BN;
    const int F = p.F, F2 = 2 * p.F;
    const int lane = threadIdx.x & 31;
    const int cta = r_local >> 7;                              // which 128-row group of the tile
    const bool grp_ok = 128 * cta < ti.rows;                   // it holds rows of this expert
    const int KG = (n_e + 127) / 128;                          // the expert's 128-row groups
    const int jb = 8 * ti.m_blk + (r_local >> 5);              // this warp's 32-row block of the expert
    // this CTA's 128 rows are row group grp0 + 2 m_blk + cta of dh's tile atoms
    const size_t g_rows = (size_t)grp0 + 2 * ti.m_blk + cta;
    // the warp's 32 rows all belong to the expert: its code tiles go by TMA
    const int w_row = r_local - lane;
    const bool tma = cs.stg != nullptr && w_row + 32 <= ti.rows;   // warp-uniform
    const int y = ti.row0 + w_row;
    float dp = 0.f;
#pragma unroll 1
    for (int it = 0; it < 4; ++it) {
      const int c = strip8(acc, half, it);
      const int col = n0 + c * 32;
      const bool live = grp_ok && col < p.N;                   // warp-uniform
      // the saved h of these 32 columns, staged in shared memory (every strip is taken,
      // live or not, so that the staging ring advances in step). Taken before the
      // tensor-memory loads: nothing may run between a tcgen05.ld and its wait that
      // could move the registers it is still filling.
      uint4 gva[4], uva[4];
      h_fetch(gva, uva);
      uint32_t v0[16], v1[16];
      tmem_ld_32x32b_x16(t_row + c * 32, v0);
      tmem_ld_32x32b_x16(t_row + c * 32 + 16, v1);
      tmem_wait_ld();
      if (it == 0) {
        tc_fence_before();
        strip_done();
      }
      if (!live) continue;
      if (!row_ok) {
#pragma unroll
        for (int i = 0; i < 4; ++i) gva[i] = uva[i] = make_uint4(0, 0, 0, 0);
      }
      float dg[32], du[32];
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(gva);
      const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(uva);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 gg2 = __bfloat1622float2(g2[i]);
        const float2 uu2 = __bfloat1622float2(u2[i]);
        const float gs[2] = {gg2.x, gg2.y}, us[2] = {uu2.x, uu2.y};
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int k = 2 * i + j;
          const float da = row_ok ? __uint_as_float(k < 16 ? v0[k] : v1[k - 16]) : 0.f;
          const float sg = sigmoid_f(gs[j]);
          const float sl = gs[j] * sg;
          dg[k] = da * pr * us[j] * (sg * (1.0f + gs[j] * (1.0f - sg)));
          du[k] = da * pr * sl;
          dp = fmaf(da, sl * us[j], dp);
        }
      }
      // along the expert's rows (warp-wide blocks): dh for the fc1 weight gradient
      uint32_t w[8];
      const size_t gcol_dh = (size_t)grp0 * (F2 / 128) + (size_t)KG * (col / 128);
      const size_t gcol_du = (size_t)grp0 * (F2 / 128) + (size_t)KG * ((F + col) / 128);
      uint32_t sc = quant_cols_warp32(dg, w, lane);
      mp.dh_cols_atoms[mma_scale_offset(gcol_dh, (col + lane) % 128, jb, 1)] = (uint8_t)sc;
      if (tma) {
        store_codes_tma(cs.stg, cs.tm_cols, col, y, w, lane);
      } else if (row_ok) {
        uint4* d = reinterpret_cast<uint4*>(mp.dh_cols + row * F2 + col);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      sc = quant_cols_warp32(du, w, lane);
      mp.dh_cols_atoms[mma_scale_offset(gcol_du, (F + col + lane) % 128, jb, 1)] = (uint8_t)sc;
      if (tma) {
        store_codes_tma(cs.stg, cs.tm_cols, F + col, y, w, lane);
      } else if (row_ok) {
        uint4* d = reinterpret_cast<uint4*>(mp.dh_cols + row * F2 + F + col);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      // along this row's columns: dh for fc1 dgrad (K = 2F); rows past the expert store
      // zero scales (their codes are never read)
      uint32_t code = quant_row32(dg, w);
      mp.dh_rows_atoms[mma_scale_offset(g_rows, r_local & 127, col / 32, F2 / 128)] = row_ok ? (uint8_t)code : 0;
      if (tma) {
        store_codes_tma(cs.stg, cs.tm_rows, col, y, w, lane);
      } else if (row_ok) {
        uint4* d = reinterpret_cast<uint4*>(mp.dh_rows + row * F2 + col);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      code = quant_row32(du, w);
      mp.dh_rows_atoms[mma_scale_offset(g_rows, r_local & 127, (F + col) / 32, F2 / 128)] = row_ok ? (uint8_t)code : 0;
      if (tma) {
        store_codes_tma(cs.stg, cs.tm_rows, F + col, y, w, lane);
      } else if (row_ok) {
        uint4* d = reinterpret_cast<uint4*>(mp.dh_rows + row * F2 + F + col);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
    if (row_ok) p.dprob_part[(long long)(2 * ti.n_blk + half) * p.M + row] = dp;
  } else if (EPI == MXEPI_DSWIGLU_F8) {
    // per-tensor FP8 fc2 dgrad: da = acc / (s_dy s_w2[e]); dg = da p u SiLU'(g),
    // du = da p SiLU(g), dp += da SiLU(g) u; dh stored in bf16 (its per-tensor scale needs
    // the max over the whole tensor, kept in amax_out)
    const float pr = (row_ok && p.probs) ? p.probs[row] : 1.0f;
    const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(p.aux);
    __nv_bfloat16* dh = reinterpret_cast<__nv_bfloat16*>(p.out2);
    const int n0 = ti.n_blk * BN;
    const float deq = mx_deq_factor(mp, ti.e);
    float dp = 0.f, amax = 0.f;
#pragma unroll 1
    for (int it = 0; it < 4; ++it) {
      const int c = strip8(acc, half, it);
      const int col = n0 + c * 32;
      const bool cols_ok = row_ok && col < p.N;
      uint4 gva[4], uva[4];
      if (cols_ok) {
        const uint4* gp = reinterpret_cast<const uint4*>(h + row * p.ld_aux + col);
        const uint4* up = reinterpret_cast<const uint4*>(h + row * p.ld_aux + p.F + col);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          gva[i] = gp[i];
          uva[i] = up[i];
        }
      }
      uint32_t v0[16], v1[16];
      tmem_ld_32x32b_x16(t_row + c * 32, v0);
      tmem_ld_32x32b_x16(t_row + c * 32 + 16, v1);
      tmem_wait_ld();
      if (it == 0) {
        tc_fence_before();
        strip_done();
      }
      if (cols_ok) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int cc = col + 16 * hh;
          const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(gva + 2 * hh);
          const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(uva + 2 * hh);
          uint4 og[2], ou[2];
          uint32_t* ogw = reinterpret_cast<uint32_t*>(og);
          uint32_t* ouw = reinterpret_cast<uint32_t*>(ou);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float2 gg2 = __bfloat1622float2(g2[i]);
            const float2 uu2 = __bfloat1622float2(u2[i]);
            const float gs[2] = {gg2.x, gg2.y}, us[2] = {uu2.x, uu2.y};
            float dg[2], du[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const float da = __uint_as_float(hh ? v1[2 * i + j] : v0[2 * i + j]) * deq;
              const float sg = sigmoid_f(gs[j]);
              const float sl = gs[j] * sg;
              dg[j] = da * pr * us[j] * (sg * (1.0f + gs[j] * (1.0f - sg)));
              du[j] = da * pr * sl;
              dp = fmaf(da, sl * us[j], dp);
            }
            ogw[i] = pack_bf16x2(dg[0], dg[1]);
            ouw[i] = pack_bf16x2(du[0], du[1]);
            // the amax of what is stored (the bf16 values the quantiser will read)
            const float2 rg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ogw[i]));
            const float2 ru = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ouw[i]));
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(rg.x), fabsf(rg.y)), fmaxf(fabsf(ru.x), fabsf(ru.y))));
          }
          uint4* d0 = reinterpret_cast<uint4*>(dh + row * p.ldo2 + cc);
          uint4* d1 = reinterpret_cast<uint4*>(dh + row * p.ldo2 + p.F + cc);
          d0[0] = og[0];
          d0[1] = og[1];
          d1[0] = ou[0];
          d1[1] = ou[1];
        }
      }
    }
    warp_amax_to(mp.amax_out, amax);
    if (row_ok) p.dprob_part[(long long)(2 * ti.n_blk + half) * p.M + row] = dp;
  } else if (EPI == MXEPI_SWIGLU_F8) {
    // per-tensor FP8 fc1: h = acc / (s_x s_w1[e]); a = SiLU(g) * u * p stored in bf16
    // (its per-tensor scale needs the max over all of a, kept in amax_out), h in bf16
    const float pr = (row_ok && p.probs) ? p.probs[row] : 1.0f;
    const int n0 = ti.n_blk * 128;
    const float deq = mx_deq_factor(mp, ti.e);
    __nv_bfloat16* a_out = reinterpret_cast<__nv_bfloat16*>(p.out);
    __nv_bfloat16* hout = reinterpret_cast<__nv_bfloat16*>(p.out2);
    float amax = 0.f;
#pragma unroll 1
    for (int it = 0; it < 2; ++it) {
      const int c = strip4(acc, half, it);
      uint32_t g0[16], g1[16], u0[16], u1[16];
      tmem_ld_32x32b_x16(t_row + c * 32, g0);
      tmem_ld_32x32b_x16(t_row + c * 32 + 16, g1);
      tmem_ld_32x32b_x16(t_row + 128 + c * 32, u0);
      tmem_ld_32x32b_x16(t_row + 128 + c * 32 + 16, u1);
      tmem_wait_ld();
      if (it == 0) {
        tc_fence_before();
        strip_done();
      }
      if (row_ok) {
        float g[32], u[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          g[i] = __uint_as_float(g0[i]) * deq;
          g[16 + i] = __uint_as_float(g1[i]) * deq;
          u[i] = __uint_as_float(u0[i]) * deq;
          u[16 + i] = __uint_as_float(u1[i]) * deq;
        }
        uint4 oa[4], hg[4], hu[4];
        uint32_t* oaw = reinterpret_cast<uint32_t*>(oa);
        uint32_t* hgw = reinterpret_cast<uint32_t*>(hg);
        uint32_t* huw = reinterpret_cast<uint32_t*>(hu);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          oaw[i] = pack_bf16x2(silu_f(g[2 * i]) * u[2 * i] * pr, silu_f(g[2 * i + 1]) * u[2 * i + 1] * pr);
          const float2 ra = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&oaw[i]));
          amax = fmaxf(amax, fmaxf(fabsf(ra.x), fabsf(ra.y)));
          hgw[i] = pack_bf16x2(g[2 * i], g[2 * i + 1]);
          huw[i] = pack_bf16x2(u[2 * i], u[2 * i + 1]);
        }
        uint4* dst = reinterpret_cast<uint4*>(a_out + row * p.ldo + n0 + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = oa[i];
        if (hout) {
          uint4* hd = reinterpret_cast<uint4*>(hout + row * p.ldo2 + n0 + c * 32);
          uint4* hd2 = reinterpret_cast<uint4*>(hout + row * p.ldo2 + p.F + n0 + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            hd[i] = hg[i];
            hd2[i] = hu[i];
          }
        }
      }
    }
    warp_amax_to(mp.amax_out, amax);
  } else {
    // ScaledSwiGLU, then MXFP8 along the output columns (one 32-column block per chunk)
    const float pr = (row_ok && p.probs) ? p.probs[row] : 1.0f;
    const int n0 = ti.n_blk * 128;
    const bool grp_ok = 128 * (r_local >> 7) < ti.rows;      // this CTA's rows hold some of the expert
    const int KG = (n_e + 127) / 128;                        // the expert's 128-row groups
    const int jb = 8 * ti.m_blk + (r_local >> 5);            // this warp's 32-row block of the expert
    uint8_t* a_codes = reinterpret_cast<uint8_t*>(p.out);
    __nv_bfloat16* hout = reinterpret_cast<__nv_bfloat16*>(p.out2);
    // a-strips in strip4 order: acc0 shares the up columns of a-strips 2 and 3, acc1 the
    // gate columns of a-strips 0 and 1, one of each per half
#pragma unroll 1
    for (int it = 0; it < 2; ++it) {
      const int c = strip4(acc, half, it);
      uint32_t g0[16], g1[16], u0[16], u1[16];
      tmem_ld_32x32b_x16(t_row + c * 32, g0);
      tmem_ld_32x32b_x16(t_row + c * 32 + 16, g1);
      tmem_ld_32x32b_x16(t_row + 128 + c * 32, u0);
      tmem_ld_32x32b_x16(t_row + 128 + c * 32 + 16, u1);
      tmem_wait_ld();
      if (it == 0) {
        tc_fence_before();
        strip_done();
      }
      if (mp.a_cols && grp_ok) {
        // training: a along the expert's rows as well, for the fc2 weight gradient (the
        // 32 lanes are 32 consecutive rows of one expert; rows past its end count as 0)
        float a[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          a[i] = row_ok ? silu_f(__uint_as_float(g0[i])) * __uint_as_float(u0[i]) * pr : 0.f;
          a[16 + i] = row_ok ? silu_f(__uint_as_float(g1[i])) * __uint_as_float(u1[i]) * pr : 0.f;
        }
        uint32_t w[8];
        const int col = n0 + c * 32;
        const uint32_t sc = quant_cols_warp32(a, w, threadIdx.x & 31);
        mp.a_cols_atoms[mma_scale_offset((size_t)grp0 * (p.N / 128) + (size_t)KG * (col / 128),
                                         (col + (threadIdx.x & 31)) % 128, jb, 1)] = (uint8_t)sc;
        if (row_ok) {
          uint4* d = reinterpret_cast<uint4*>(mp.a_cols + row * p.N + col);
          d[0] = make_uint4(w[0], w[1], w[2], w[3]);
          d[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
      if (row_ok) {
        float a[32];
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          a[i] = silu_f(__uint_as_float(g0[i])) * __uint_as_float(u0[i]) * pr;
          a[16 + i] = silu_f(__uint_as_float(g1[i])) * __uint_as_float(u1[i]) * pr;
          amax = fmaxf(amax, fmaxf(fabsf(a[i]), fabsf(a[16 + i])));
        }
        const int bexp = (int)((__float_as_uint(amax) >> 23) & 0xFF);
        const int code = max(bexp - 8, 0);
        const float inv = __uint_as_float((uint32_t)(254 - code) << 23);
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] *= inv;
        uint32_t w0[4], w1[4];
        pack_e4m3x16(a, w0);
        pack_e4m3x16(a + 16, w1);
        uint4* dst = reinterpret_cast<uint4*>(a_codes + row * p.ldo + n0 + c * 32);
        dst[0] = make_uint4(w0[0], w0[1], w0[2], w0[3]);
        dst[1] = make_uint4(w1[0], w1[1], w1[2], w1[3]);
        sc_word |= (uint32_t)code << (8 * c);
        if (hout) {
          uint4 hg[4], hu[4];
          uint32_t* hgw = reinterpret_cast<uint32_t*>(hg);
          uint32_t* huw = reinterpret_cast<uint32_t*>(hu);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            hgw[i] = pack_bf16x2(__uint_as_float(g0[2 * i]), __uint_as_float(g0[2 * i + 1]));
            hgw[8 + i] = pack_bf16x2(__uint_as_float(g1[2 * i]), __uint_as_float(g1[2 * i + 1]));
            huw[i] = pack_bf16x2(__uint_as_float(u0[2 * i]), __uint_as_float(u0[2 * i + 1]));
            huw[8 + i] = pack_bf16x2(__uint_as_float(u1[2 * i]), __uint_as_float(u1[2 * i + 1]));
          }
          uint4* hd = reinterpret_cast<uint4*>(hout + row * p.ldo2 + n0 + c * 32);
          uint4* hd2 = reinterpret_cast<uint4*>(hout + row * p.ldo2 + p.F + n0 + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            hd[i] = hg[i];
            hd2[i] = hu[i];
          }
        }
      }
    }
  }
  return sc_word;
}

}  // namespace moe
