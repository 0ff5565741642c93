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
//   * the MMA thread moves the atoms into tensor memory with tcgen05.cp (32 lanes x 16 B,
//     replicated to the four sub-partitions), then issues the four K=32 MMAs of the
//     k-block, selecting scale byte kk of each word through the scale-factor ids;
//   * two 256-column accumulators plus 12 scale columns exceed the 512 tensor-memory
//     columns, so the accumulators overlap: acc0 = columns [0, 256), acc1 = [224, 480),
//     scales at [480, 492). The epilogue drains the shared 32-column strip first and
//     signals `tovl`; the next tile's MMAs wait for that strip (and for the full drain
//     of the tile two back) instead of the whole previous epilogue.
#pragma once
#include "grouped_gemm_sm100.cuh"
#include "token_kernels.cuh"

namespace moe {

namespace mx {
// tensor-memory layout shared by the MXFP8 pair kernels (columns of each CTA's 512)
constexpr int BN = 256;                       // accumulator columns per tile
constexpr uint32_t kAcc1Col = 224;            // acc0 = [0, 256), acc1 = [224, 480)
constexpr uint32_t kSfaCol = 480;             // A scales: 4 columns
constexpr uint32_t kSfbCol = 484;             // B scales: 2 x 4 columns
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

// E4M3 codes of 32 fp32 values (one lane's row) quantised along the 32 LANES of the warp:
// for each column j the block maximum is the warp-wide max of |v[j]| (one redux: the bits
// of a non-negative float order like the float), E8M0 code max(exp(amax) - 8, 0), element
// scaled by 2^(127 - code) exactly and rounded to nearest even with saturation. Lanes
// that hold no row pass zeros. Every lane of the warp must call this together. Returns
// the codes in `w` (byte j = column j) and, in lane j, the scale code of column j.
__device__ __forceinline__ uint32_t quant_cols_warp32(const float (&v)[32], uint32_t (&w)[8], int lane) {
  uint32_t mine = 0;
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const uint32_t m0 = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v[j])));
    const uint32_t m1 = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v[j + 1])));
    const int c0 = max((int)(m0 >> 23) - 8, 0), c1 = max((int)(m1 >> 23) - 8, 0);
    const float i0 = __uint_as_float((uint32_t)(254 - c0) << 23), i1 = __uint_as_float((uint32_t)(254 - c1) << 23);
    const uint32_t pair =
        (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(v[j] * i0, v[j + 1] * i1), __NV_SATFINITE, __NV_E4M3);
    if ((j & 2) == 0)
      w[j >> 2] = pair;
    else
      w[j >> 2] |= pair << 16;
    if (lane == j) mine = (uint32_t)c0;
    if (lane == j + 1) mine = (uint32_t)c1;
  }
  return mine;
}

// E4M3 codes of 32 fp32 values of one row quantised as one block along the row; returns
// the block's scale code.
__device__ __forceinline__ uint32_t quant_row32(float (&v)[32], uint32_t (&w)[8]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int code = max((int)((__float_as_uint(amax) >> 23) & 0xFF) - 8, 0);
  const float inv = __uint_as_float((uint32_t)(254 - code) << 23);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] *= inv;
  pack_e4m3x16(v, *reinterpret_cast<uint32_t(*)[4]>(&w[0]));
  pack_e4m3x16(v + 16, *reinterpret_cast<uint32_t(*)[4]>(&w[4]));
  return (uint32_t)code;
}

// Drains one 128-row x 256-column accumulator (this thread's row: lane quadrant of
// `t_row`, row r_local of the output tile) and runs the epilogue EPI on it. The 32-column
// strip that acc0 and acc1 share is drained first by its owning half, which then calls
// `strip_done()`; the other half calls it before reading anything (warp-uniform calls, so
// the callee may signal once per warp). Returns the SwiGLU_Q row's four scale bytes.
// DSWIGLU also takes the expert's first 128-row group (grp0: groups of earlier experts),
// its row count n_e, which place its scale atoms, and `h_fetch(g, u)`, which hands this
// thread the saved h of its row for the next 32-column strip in the order the strips are
// drained (the caller stages h in shared memory ahead of the epilogue).
struct NoHFetch {
  __device__ bool operator()(uint4 (&)[4], uint4 (&)[4]) const { return false; }
};

template <int EPI, class StripDone, class HFetch = NoHFetch>
__device__ __forceinline__ uint32_t mxf8_epilogue_tile(const MxGemmParams& mp, const TileInfo& ti, uint32_t t_row,
                                                       int acc, int half, int r_local, int tile_bm,
                                                       StripDone&& strip_done, int grp0 = 0, int n_e = 0,
                                                       const HFetch& h_fetch = HFetch{}) {
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
    // the 32-column strip shared with the other accumulator: chunk 7 of acc0 (upper
    // half), chunk 0 of acc1 (lower half); its owner drains it first, then signals
    const bool owner = acc ? (half == 0) : (half == 1);
    if (!owner) strip_done();
    const float deq = mx_deq_factor(mp, EPI == MXEPI_WGRAD ? 0 : ti.e);
#pragma unroll 1
    for (int it = 0; it < 4; ++it) {
      const int c = owner ? (acc ? it : (it == 0 ? 7 : 3 + it)) : 4 * half + it;
      uint32_t v0[16], v1[16];
      tmem_ld_32x32b_x16(t_row + c * 32, v0);
      tmem_ld_32x32b_x16(t_row + c * 32 + 16, v1);
      tmem_wait_ld();
      if (owner && it == 0) {
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
    const bool half_ok = n0 + 128 * half < p.N;                // F % 128 == 0: halves are whole
    const bool live = grp_ok && half_ok;                       // warp-uniform
    const int KG = (n_e + 127) / 128;                          // the expert's 128-row groups
    const int jb = 8 * ti.m_blk + (r_local >> 5);              // this warp's 32-row block of the expert
    const bool owner = acc ? (half == 0) : (half == 1);
    if (!owner) strip_done();
    float dp = 0.f;
    uint32_t sg_word = 0, su_word = 0;   // this row's scale codes of its four dg / du blocks
#pragma unroll 1
    for (int it = 0; it < 4; ++it) {
      const int c = owner ? (acc ? it : (it == 0 ? 7 : 3 + it)) : 4 * half + it;
      const int col = n0 + c * 32;
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
      if (owner && it == 0) {
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
      if (row_ok) {
        uint4* d = reinterpret_cast<uint4*>(mp.dh_cols + row * F2 + col);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      sc = quant_cols_warp32(du, w, lane);
      mp.dh_cols_atoms[mma_scale_offset(gcol_du, (F + col + lane) % 128, jb, 1)] = (uint8_t)sc;
      if (row_ok) {
        uint4* d = reinterpret_cast<uint4*>(mp.dh_cols + row * F2 + F + col);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      // along this row's columns: dh for fc1 dgrad (K = 2F)
      sg_word |= quant_row32(dg, w) << (8 * (c & 3));
      if (row_ok) {
        uint4* d = reinterpret_cast<uint4*>(mp.dh_rows + row * F2 + col);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      su_word |= quant_row32(du, w) << (8 * (c & 3));
      if (row_ok) {
        uint4* d = reinterpret_cast<uint4*>(mp.dh_rows + row * F2 + F + col);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
    if (live) {
      // this CTA's 128 rows are row group grp0 + 2 m_blk + cta of dh's tile atoms; rows
      // past the expert store zero scales (their codes are never read)
      const size_t g = (size_t)grp0 + 2 * ti.m_blk + cta;
      const int kb_g = (n0 + 128 * half) / 32, kb_u = (F + n0 + 128 * half) / 32;
      *reinterpret_cast<uint32_t*>(mp.dh_rows_atoms + mma_scale_offset(g, r_local & 127, kb_g, F2 / 128)) =
          row_ok ? sg_word : 0u;
      *reinterpret_cast<uint32_t*>(mp.dh_rows_atoms + mma_scale_offset(g, r_local & 127, kb_u, F2 / 128)) =
          row_ok ? su_word : 0u;
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
    const bool owner = acc ? (half == 0) : (half == 1);
    if (!owner) strip_done();
    float dp = 0.f, amax = 0.f;
#pragma unroll 1
    for (int it = 0; it < 4; ++it) {
      const int c = owner ? (acc ? it : (it == 0 ? 7 : 3 + it)) : 4 * half + it;
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
      if (owner && it == 0) {
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
    const bool owner = acc ? (half == 0) : (half == 1);
    if (!owner) strip_done();
    float amax = 0.f;
#pragma unroll 1
    for (int it = 0; it < 2; ++it) {
      const int c = owner ? (acc ? it : 3 - it) : 2 * half + it;
      uint32_t g0[16], g1[16], u0[16], u1[16];
      tmem_ld_32x32b_x16(t_row + c * 32, g0);
      tmem_ld_32x32b_x16(t_row + c * 32 + 16, g1);
      tmem_ld_32x32b_x16(t_row + 128 + c * 32, u0);
      tmem_ld_32x32b_x16(t_row + 128 + c * 32 + 16, u1);
      tmem_wait_ld();
      if (owner && it == 0) {
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
    // output chunk 3 of acc0 (its up columns are the shared strip) belongs to the
    // upper half, chunk 0 of acc1 (gate columns) to the lower half
    const bool owner = acc ? (half == 0) : (half == 1);
    if (!owner) strip_done();
#pragma unroll 1
    for (int it = 0; it < 2; ++it) {
      const int c = owner ? (acc ? it : 3 - it) : 2 * half + it;
      uint32_t g0[16], g1[16], u0[16], u1[16];
      tmem_ld_32x32b_x16(t_row + c * 32, g0);
      tmem_ld_32x32b_x16(t_row + c * 32 + 16, g1);
      tmem_ld_32x32b_x16(t_row + 128 + c * 32, u0);
      tmem_ld_32x32b_x16(t_row + 128 + c * 32 + 16, u1);
      tmem_wait_ld();
      if (owner && it == 0) {
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
