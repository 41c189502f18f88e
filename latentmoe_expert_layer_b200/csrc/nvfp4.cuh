// NVFP4 quantisation: E2M1 elements in 16-element blocks along the reduction dimension, one E4M3
// scale per block, one fp32 scale per tensor.  The pages name the two-level scheme (a per-tensor
// global scale and per-block fine scales: "Nemotron 3 Super" notes, section 3.6; E2M1 data with E4M3
// block scales: "Nemotron 3 Ultra" summary) but fix neither block size nor rounding.  This library
// uses 16-element blocks and round-to-nearest-even with saturation, every decision in fp32:
//
//   g   = amax(tensor) / 2688            (2688 = 6 * 448; an all-zero tensor gets g = 1)
//   s   = E4M3_rne_sat( amax(block) / (6 g) )
//   q_i = E2M1_rne_sat( v_i / (s g) )     (s decoded to fp32 first; s == 0 gives q_i = sign only)
//
// Layouts
//   codes   row-major [rows, K/2] bytes, element 2i in the low nibble, 2i+1 in the high nibble
//   weight scales: 512-byte atoms, one per (128 rows, 64 K) tile; inside an atom the scale of row r
//           (0..127) and K-block s (0..3) sits at byte (r % 32) * 16 + (r / 32) * 4 + s, which is the
//           layout tcgen05.cp (32x128b, replicated to the 4 lane quadrants) turns into the TMEM scale
//           columns the block-scaled MMA reads.  Atoms are ordered [row tile][K atom], K atoms padded
//           to a multiple of 4 (one 256-element pipeline stage) with zero scales.
//   activation scales: tile-local atoms (see act_sf_offset), so that one token tile's scales for one
//           pipeline stage are a single contiguous copy.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "ptx.cuh"

namespace lmoe {

constexpr float NVFP4_TENSOR_DIV = 2688.0f;  // E2M1 max (6) times E4M3 max (448)
constexpr int NVFP4_STAGE_K = 256;           // FP4 elements per 128-byte smem row

// E2M1 code of r: magnitude rounded to {0, .5, 1, 1.5, 2, 3, 4, 6} (nearest, ties to the even
// code, saturating at 6); bit 3 carries the sign of r.
__device__ __forceinline__ uint32_t e2m1_code(float r) {
  const float a = fabsf(r);
  uint32_t c;
  if (a <= 0.25f) c = 0u;
  else if (a < 0.75f) c = 1u;
  else if (a <= 1.25f) c = 2u;
  else if (a < 1.75f) c = 3u;
  else if (a <= 2.5f) c = 4u;
  else if (a < 3.5f) c = 5u;
  else if (a <= 5.0f) c = 6u;
  else c = 7u;
  return c | ((__float_as_uint(r) >> 28) & 8u);
}

__device__ __forceinline__ uint32_t e4m3_rne_sat(float s) {
  return (uint32_t)__nv_cvt_float_to_fp8(s, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3);
  return __half2float(__half(h));
}

__device__ __forceinline__ float tensor_scale_from_amax(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, NVFP4_TENSOR_DIV) : 1.0f;
}

// Quantise one 16-element block with tensor scale g.  Returns the E4M3 scale byte; writes the 8
// packed code bytes (element 2i low nibble) into codes[0..1] (two 32-bit words).
__device__ __forceinline__ uint32_t nvfp4_block(const float (&v)[16], float g, uint32_t (&codes)[2]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float den6 = __fmul_rn(6.0f, g);
  const uint32_t sb = e4m3_rne_sat(__fdiv_rn(amax, den6));
  const float den = __fmul_rn(e4m3_to_f32(sb), g);
  codes[0] = codes[1] = 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t c = den > 0.f ? e2m1_code(__fdiv_rn(v[i], den)) : ((__float_as_uint(v[i]) >> 28) & 8u);
    codes[i >> 3] |= c << (4 * (i & 7));
  }
  return sb;
}

// Signed value of a 4-bit E2M1 code.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t m = c & 7u;
  const float a = m < 4u ? 0.5f * (float)m : (m == 4u ? 2.0f : m == 5u ? 3.0f : m == 6u ? 4.0f : 6.0f);
  return (c & 8u) ? -a : a;
}

// Sum of squared reconstruction errors of a block under block scale s (decoded E4M3) and tensor
// scale g: every step rounded to fp32 on its own (no fused multiply-add), elements in order.
__device__ __forceinline__ float nvfp4_block_sq_error(const float (&v)[16], float s, float g) {
  const float den = __fmul_rn(s, g);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float q = den > 0.f ? e2m1_value(e2m1_code(__fdiv_rn(v[i], den))) : 0.f;
    const float e = __fsub_rn(v[i], __fmul_rn(__fmul_rn(q, s), g));
    acc = __fadd_rn(acc, __fmul_rn(e, e));
  }
  return acc;
}

// nvfp4_block with the block scale searched for the smallest squared error: candidates c0 (the
// amax rule), c0 + 1, c0 - 1 .. c0 - 6 (inside the positive finite codes 1..0x7E); the first
// strict minimum wins.
__device__ __forceinline__ uint32_t nvfp4_block_mse(const float (&v)[16], float g, uint32_t (&codes)[2]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t c0 = e4m3_rne_sat(__fdiv_rn(amax, __fmul_rn(6.0f, g)));
  uint32_t best = c0;
  float best_e = nvfp4_block_sq_error(v, e4m3_to_f32(c0), g);
#pragma unroll 1
  for (int t = 0; t < 7; ++t) {
    const int c = (int)c0 + (t == 0 ? 1 : -t);
    if (c < 1 || c > 0x7E) continue;
    const float e = nvfp4_block_sq_error(v, e4m3_to_f32((uint32_t)c), g);
    if (e < best_e) {
      best_e = e;
      best = (uint32_t)c;
    }
  }
  const float den = __fmul_rn(e4m3_to_f32(best), g);
  codes[0] = codes[1] = 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t c = den > 0.f ? e2m1_code(__fdiv_rn(v[i], den)) : ((__float_as_uint(v[i]) >> 28) & 8u);
    codes[i >> 3] |= c << (4 * (i & 7));
  }
  return best;
}

// Eight E2M1 codes (element 2i in the low nibble) of v[i] * rcp, rounded to nearest even and
// saturated by the hardware conversion.
__device__ __forceinline__ uint32_t e2m1x8_scaled(const float* v, float rcp) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(__fmul_rn(v[0], rcp)), "f"(__fmul_rn(v[1], rcp)), "f"(__fmul_rn(v[2], rcp)), "f"(__fmul_rn(v[3], rcp)),
        "f"(__fmul_rn(v[4], rcp)), "f"(__fmul_rn(v[5], rcp)), "f"(__fmul_rn(v[6], rcp)), "f"(__fmul_rn(v[7], rcp)));
  return r;
}

// Eight E2M1 codes of r[0..7] (already divided by the block scale), hardware conversion: round to
// nearest even, saturating at 6.
__device__ __forceinline__ uint32_t e2m1x8(const float* r) {
  uint32_t o;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(o)
      : "f"(r[0]), "f"(r[1]), "f"(r[2]), "f"(r[3]), "f"(r[4]), "f"(r[5]), "f"(r[6]), "f"(r[7]));
  return o;
}

// Quantiser for bf16 activations (x, h): the oracle's decisions exactly (IEEE division of each
// element by the decoded block scale, then round-to-nearest-even).  bf16 inputs hit exact E2M1
// rounding ties often enough that a reciprocal multiply would land beside them; the rounding itself
// is the hardware conversion.  A zero block scale gives zero codes.
__device__ __forceinline__ uint32_t nvfp4_block_exact(const float (&v)[16], float g, uint32_t (&codes)[2]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t sb = e4m3_rne_sat(__fdiv_rn(amax, __fmul_rn(6.0f, g)));
  const float den = __fmul_rn(e4m3_to_f32(sb), g);
  float r[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) r[i] = den > 0.f ? __fdiv_rn(v[i], den) : 0.f;
  codes[0] = e2m1x8(r);
  codes[1] = e2m1x8(r + 8);
  return sb;
}

// Activation block quantiser for fp32 accumulator outputs (u, u_s in the GEMM epilogue): same scale
// rule, elements scaled by the fp32 reciprocal of the block scale (one multiply and half a conversion
// per element).  fp32 accumulator values essentially never sit on an E2M1 rounding tie.
__device__ __forceinline__ uint32_t nvfp4_block_fast(const float (&v)[16], float g, uint32_t (&codes)[2]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t sb = e4m3_rne_sat(__fdiv_rn(amax, __fmul_rn(6.0f, g)));
  const float den = __fmul_rn(e4m3_to_f32(sb), g);
  const float rcp = den > 0.f ? __frcp_rn(den) : 0.f;
  codes[0] = e2m1x8_scaled(v, rcp);
  codes[1] = e2m1x8_scaled(v + 8, rcp);
  return sb;
}

// Activation scales live in tile-local atoms, so that the GEMM fetches one token tile's scales for one
// pipeline stage with a single bulk copy: for token tile `tile` (nra = ceil(tile tokens / 128) row
// atoms) and stage `st` (256 K elements = 4 K atoms of 64), the 4 * nra atoms are contiguous, K-atom
// major: atom (ka, ra) at ((tile * stages + st) * 4 + ka) * nra + ra.  Inside an atom the layout is the
// weight atoms' one.  Each K atom's scales must start on a 4-column-aligned TMEM address for the
// block-scaled MMA, hence one atom (one tcgen05.cp) per K atom and 128 tokens even for short tiles.
__host__ __device__ __forceinline__ long long act_sf_offset(long long tile, int j, int kb16, int stages, int nra,
                                                           int rep = 0, int reps = 1) {
  const int st = kb16 >> 4, ka = (kb16 >> 2) & 3, s = kb16 & 3;
  // reps > 1: every atom stored `reps` times in a row (copy `rep` here), as for the weight scales
  return (((((tile * stages + st) * 4 + ka) * nra + (j >> 7)) * reps) + rep) * 512 + (j & 31) * 16 +
         ((j & 127) >> 5) * 4 + s;
}

// Weight-scale atoms are stored replicated: each 512-byte atom four times in a row (2 KB), the
// image tcgen05.cp.128x256b turns into the scale columns of all four TMEM lane quadrants (lane L
// reads bytes 16 L .. 16 L + 15 of the 2 KB block), so one copy instruction moves two K atoms.
constexpr int SF_WREP = 4;

// Byte offset of the scale of (row r, 16-element block kb), copy `rep` (0..3), inside a
// weight-scale array with `atoms_k` K atoms per 128-row tile.
__host__ __device__ __forceinline__ long long sf_atom_offset(long long r, int kb, int atoms_k, int rep = 0) {
  return ((r >> 7) * atoms_k + (kb >> 2)) * (512 * SF_WREP) + rep * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 +
         (kb & 3);
}

__host__ __device__ __forceinline__ int sf_atoms_k(int K) { return ((K + NVFP4_STAGE_K - 1) / NVFP4_STAGE_K) * 4; }
__host__ __device__ __forceinline__ int act_sf_pitch(int K) { return ((K + NVFP4_STAGE_K - 1) / NVFP4_STAGE_K) * 16; }

// ------------------------------------------------------------------------------------------------
// amax of contiguous groups (one weight matrix each): amax_bits[blockIdx.y] = max |w| over the
// group's group_elems bf16 values (fp32 bits; non-negative floats order like unsigned ints).
// ------------------------------------------------------------------------------------------------
__global__ void amax_groups_kernel(const __nv_bfloat16* __restrict__ w, long long group_elems,
                                   unsigned* __restrict__ amax_bits) {
  const uint4* base = reinterpret_cast<const uint4*>(w + (long long)blockIdx.y * group_elems);
  const long long n8 = group_elems / 8;
  float m = 0.f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const uint4 q = base[i];
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(p[j]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0 && m > 0.f) atomicMax(&amax_bits[blockIdx.y], __float_as_uint(m));
}

// ------------------------------------------------------------------------------------------------
// Weight quantiser: one thread per 16-element block.  Writes codes [rows, K/2], scales into atoms,
// and (thread 0 of each group) the group's fp32 tensor scale.  mse: block scales by nvfp4_block_mse.
// ------------------------------------------------------------------------------------------------
__global__ void quant_weight_kernel(const __nv_bfloat16* __restrict__ w, long long rows, int K, long long rows_per_group,
                                   const unsigned* __restrict__ amax_bits, uint8_t* __restrict__ codes,
                                   uint8_t* __restrict__ sf_atoms, float* __restrict__ g_out, int mse) {
  const int nb = K / 16;
  const long long total = rows * nb;
  const int atoms_k = sf_atoms_k(K);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / nb;
    const int kb = (int)(i - r * nb);
    const long long grp = r / rows_per_group;
    const float g = tensor_scale_from_amax(__uint_as_float(amax_bits[grp]));
    const uint4* src = reinterpret_cast<const uint4*>(w + r * K + kb * 16);
    float v[16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 q = src[h];
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(p[j]);
        v[h * 8 + 2 * j] = f.x;
        v[h * 8 + 2 * j + 1] = f.y;
      }
    }
    uint32_t c[2];
    const uint32_t sb = mse ? nvfp4_block_mse(v, g, c) : nvfp4_block(v, g, c);
    *reinterpret_cast<uint2*>(codes + r * (K / 2) + kb * 8) = make_uint2(c[0], c[1]);
#pragma unroll
    for (int rp = 0; rp < SF_WREP; ++rp) sf_atoms[sf_atom_offset(r, kb, atoms_k, rp)] = (uint8_t)sb;
    if (kb == 0 && r % rows_per_group == 0) g_out[grp] = g;
  }
}

// ------------------------------------------------------------------------------------------------
// Activation amax: amax_bits[0] = max |a| over a bf16 [rows, K] tensor.
// ------------------------------------------------------------------------------------------------
__global__ void amax_act_kernel(const __nv_bfloat16* __restrict__ a, long long n_vec8, unsigned* __restrict__ amax_bits) {
  float m = 0.f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec8;
       i += (long long)gridDim.x * blockDim.x) {
    const uint4 q = reinterpret_cast<const uint4*>(a)[i];
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(p[j]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0 && m > 0.f) atomicMax(amax_bits, __float_as_uint(m));
}

// ------------------------------------------------------------------------------------------------
// Activation quantiser.  Output row r (0..n_rows) reads source row (src_rows ? src_rows[r] : r) and
// is written as codes [n_rows, K/2] plus scales in tile-local atoms.  Token tiles: dense mode
// (offsets == nullptr) tile = r / tile_rows; grouped mode the tiles restart at each expert's first
// row: expert e = the one with offsets[e] <= r < offsets[e + 1], tile = tile0[e] + (r - offsets[e])
// / tile_rows.  nra == 0: scales in plain row-major bytes [n_rows, K/16] instead of atoms.  One
// thread per 16-element block; tensor scale from amax_bits[0], also written to *g_out.
// ------------------------------------------------------------------------------------------------
// Loads of routing maps and activations in the shared device functions below.  SAME_LAUNCH: the
// data was written earlier in the same launch by other blocks (the fused decode routing), so it is
// read through L2 only; otherwise it is read-only for the kernel and may be cached on the SM.
template <bool SAME_LAUNCH, typename V>
__device__ __forceinline__ V ld_act(const V* p) {
  if constexpr (SAME_LAUNCH) return __ldcg(p);
  else return __ldg(p);
}

// The blocks i = i0, i0 + stride, ... of quant_act_kernel (shared with the fused decode routing).
template <bool SAME_LAUNCH>
__device__ __forceinline__ void quant_act_blocks(const __nv_bfloat16* __restrict__ a, int K,
                                                 const int* __restrict__ src_rows, long long n_rows, int n_src_rows,
                                                 const int* __restrict__ offsets, const int* __restrict__ tile0,
                                                 int n_experts, int tile_rows, int nra, float g,
                                                 uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                 unsigned* status, int reps, long long i0, long long stride) {
  const int nb = K / 16;
  const int stages = (K + NVFP4_STAGE_K - 1) / NVFP4_STAGE_K;
  const long long total = n_rows * nb;
  for (long long i = i0; i < total; i += stride) {
    const long long r = i / nb;
    const int kb = (int)(i - r * nb);
    long long sr = r;
    if (src_rows) {
      sr = src_rows[r];
      if (sr < 0 || sr >= n_src_rows) {
        atomicOr(status, DEV_STATUS_BAD_INDEX);
        continue;
      }
    }
    long long tile;
    int j;  // row within the tile
    if (offsets) {
      int lo = 0, hi = n_experts - 1;  // largest expert whose first row is <= r
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offsets[mid] <= r) lo = mid;
        else hi = mid - 1;
      }
      const int local = (int)(r - offsets[lo]);
      tile = tile0[lo] + local / tile_rows;
      j = local % tile_rows;
    } else {
      tile = r / tile_rows;
      j = (int)(r % tile_rows);
    }
    const uint4* src = reinterpret_cast<const uint4*>(a + sr * K + kb * 16);
    float v[16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 q = ld_act<SAME_LAUNCH>(src + h);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 f = __bfloat1622float2(p[t]);
        v[h * 8 + 2 * t] = f.x;
        v[h * 8 + 2 * t + 1] = f.y;
      }
    }
    uint32_t c[2];
    const uint32_t sb = nvfp4_block_exact(v, g, c);
    *reinterpret_cast<uint2*>(codes + r * (K / 2) + kb * 8) = make_uint2(c[0], c[1]);
    if (nra > 0) {
      for (int rp = 0; rp < reps; ++rp) sf[act_sf_offset(tile, j, kb, stages, nra, rp, reps)] = (uint8_t)sb;
    }
    else sf[r * nb + kb] = (uint8_t)sb;  // plain row-major scales
  }
}

__global__ void quant_act_kernel(const __nv_bfloat16* __restrict__ a, int K, const int* __restrict__ src_rows,
                                 long long n_rows, int n_src_rows, const int* __restrict__ offsets,
                                 const int* __restrict__ tile0, int n_experts, int tile_rows, int nra,
                                 const unsigned* __restrict__ amax_bits, uint8_t* __restrict__ codes,
                                 uint8_t* __restrict__ sf, float* __restrict__ g_out, unsigned* status, int reps) {
  const float g = tensor_scale_from_amax(__uint_as_float(amax_bits[0]));
  if (blockIdx.x == 0 && threadIdx.x == 0 && g_out) *g_out = g;
  quant_act_blocks<false>(a, K, src_rows, n_rows, n_src_rows, offsets, tile0, n_experts, tile_rows, nra, g, codes, sf,
                          status, reps, (long long)blockIdx.x * blockDim.x + threadIdx.x,
                          (long long)gridDim.x * blockDim.x);
}

// ------------------------------------------------------------------------------------------------
// Grouped copy of per-token NVFP4 rows: grouped row r gets the codes of token tok_of_row[r]
// (quantised once per token: a row's codes and block scales depend only on its values and the
// tensor scale) and its block scales go into the consuming GEMM's tile-local atoms.  One warp per
// row; K is a multiple of 128, so a row is a whole number of 512-byte code chunks and 4-byte scale
// groups, and the four scales of one K atom of a row are four adjacent bytes of the atom.
// ------------------------------------------------------------------------------------------------
// Rows r = r0, r0 + stride, ... of gather_act_q_kernel, one per warp (shared with the fused decode
// routing, which wrote the routing maps and the per-token codes earlier in the same launch).
// MAPS_SMEM: offsets and tile0 point to copies in shared memory (the per-row expert search then
// costs no memory round trips).
template <bool SAME_LAUNCH, bool MAPS_SMEM = false>
__device__ __forceinline__ void gather_act_q_rows(const uint8_t* __restrict__ codes_tok,
                                                  const uint8_t* __restrict__ sf_tok, int K,
                                                  const int* __restrict__ tok_of_row, long long n_rows, int n_tok,
                                                  const int* __restrict__ offsets, const int* __restrict__ tile0,
                                                  int n_experts, int tile_rows, int nra, uint8_t* __restrict__ codes,
                                                  uint8_t* __restrict__ sf, unsigned* status, int reps, long long r0,
                                                  long long stride) {
  const int lane = threadIdx.x & 31;
  const int row_bytes = K / 2, nb = K / 16;
  const int stages = (K + NVFP4_STAGE_K - 1) / NVFP4_STAGE_K;
  for (long long r = r0; r < n_rows; r += stride) {
    const int t = ld_act<SAME_LAUNCH>(tok_of_row + r);
    if (t < 0 || t >= n_tok) {
      if (lane == 0) atomicOr(status, DEV_STATUS_BAD_INDEX);
      continue;
    }
    int lo = 0, hi = n_experts - 1;  // largest expert whose first row is <= r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((MAPS_SMEM ? offsets[mid] : ld_act<SAME_LAUNCH>(offsets + mid)) <= r) lo = mid;
      else hi = mid - 1;
    }
    const int local = (int)(r - (MAPS_SMEM ? offsets[lo] : ld_act<SAME_LAUNCH>(offsets + lo)));
    const long long tile = (MAPS_SMEM ? tile0[lo] : ld_act<SAME_LAUNCH>(tile0 + lo)) + local / tile_rows;
    const int j = local % tile_rows;
    for (int c = lane * 16; c < row_bytes; c += 32 * 16)
      *reinterpret_cast<uint4*>(codes + r * row_bytes + c) =
          ld_act<SAME_LAUNCH>(reinterpret_cast<const uint4*>(codes_tok + (long long)t * row_bytes + c));
    for (int q = lane; q < nb / 4; q += 32) {
      const uint32_t v = ld_act<SAME_LAUNCH>(reinterpret_cast<const unsigned int*>(sf_tok + (long long)t * nb + 4 * q));
      for (int rp = 0; rp < reps; ++rp)
        *reinterpret_cast<uint32_t*>(sf + act_sf_offset(tile, j, 4 * q, stages, nra, rp, reps)) = v;
    }
  }
}

__global__ void __launch_bounds__(256)
    gather_act_q_kernel(const uint8_t* __restrict__ codes_tok, const uint8_t* __restrict__ sf_tok, int K,
                        const int* __restrict__ tok_of_row, long long n_rows, int n_tok,
                        const int* __restrict__ offsets, const int* __restrict__ tile0, int n_experts, int tile_rows,
                        int nra, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, unsigned* status,
                        int reps) {
  gather_act_q_rows<false>(codes_tok, sf_tok, K, tok_of_row, n_rows, n_tok, offsets, tile0, n_experts, tile_rows, nra,
                           codes, sf, status, reps, ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5,
                    ((long long)gridDim.x * blockDim.x) >> 5);
}

}  // namespace lmoe
