// Routing, dispatch grouping and combine kernels of the LatentMoE layer.
//
// Router + top-K: the gating network scores every token in the full model dimension d and keeps the
// K best of N experts ("Nemotron 3 Super" notes, section 3.1 table: top-22 of 512; section 3.2: the
// gating network stays in dimension d).  The gate is the softmax over the K selected logits.
//
// Dispatch: the (token, slot) assignments are grouped by expert with a histogram and an exclusive
// prefix sum, so that the latent rows h[t] sent to one expert sit contiguously ("the compressed
// representation is routed to the expanded expert set", section 3.2).  The grouping is stable in
// (token, slot) order, which makes every map (row_of, tok_of_row) uniquely defined.
//
// Combine: z[t] = sum_k o[row_of[t, k]], in slot order, fp32 accumulation (the gate is already
// folded into o by the second expert GEMM's epilogue).
#pragma once
#include <cuda_bf16.h>
#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace lmoe {

// ------------------------------------------------------------------------------------------------
// fp32 router (used when the router weights are kept in fp32): logits[t, e] = x[t, :] . W_r[e, :]
// one block per token; x row staged in shared memory; one warp per expert, lanes stride over d.
// ------------------------------------------------------------------------------------------------
__global__ void router_f32_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ w, int d,
                                  int n_experts, float* __restrict__ logits) {
  extern __shared__ float xs[];
  const int t = blockIdx.x;
  for (int j = threadIdx.x; j < d; j += blockDim.x) xs[j] = __bfloat162float(x[(long long)t * d + j]);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int e = warp; e < n_experts; e += nw) {
    const float* we = w + (long long)e * d;
    float acc = 0.f;
    for (int j = lane; j < d; j += 32) acc = fmaf(xs[j], we[j], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) logits[(long long)t * n_experts + e] = acc;
  }
}

// ------------------------------------------------------------------------------------------------
// top-K + softmax + per-chunk expert histogram.  One block per chunk of `chunk_tokens` consecutive
// tokens, one warp per token.  Lane j holds the candidates j, j + 32, ... (P of them); it sorts them
// once (bitonic network in registers, order: value desc, index asc).  Then K rounds of a warp
// arg-max over the lanes' current heads pick the experts in output order; only the lane that owned
// the winner shifts its sorted list by one.  Requires K <= 32 and N <= 32 * P.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

template <int P>
__global__ void __launch_bounds__(1024)
    topk_hist_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T, int n_experts,
                     int k, int chunk_tokens, int* __restrict__ topk_idx, float* __restrict__ topk_gate,
                     int* __restrict__ chunk_counts) {
  extern __shared__ int s_counts[];  // [n_experts]
  for (int e = threadIdx.x; e < n_experts; e += blockDim.x) s_counts[e] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int t_begin = blockIdx.x * chunk_tokens;
  const int t_end = min(T, t_begin + chunk_tokens);
  for (int t = t_begin + warp; t < t_end; t += nwarps) {
    const float* lrow = logits + (long long)t * n_experts;
    float v[P];
    int ix[P];
#pragma unroll
    for (int i = 0; i < P; ++i) {
      const int e = i * 32 + lane;
      const bool ok = e < n_experts;
      v[i] = ok ? lrow[e] + (bias ? bias[e] : 0.f) : -INFINITY;
      ix[i] = ok ? e : 0x7fffffff;
    }
#pragma unroll
    for (int size = 2; size <= P; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
        for (int i = 0; i < P; ++i) {
          const int j = i ^ stride;
          if (j > i) {
            const bool desc = (i & size) == 0;
            const bool sw = desc ? better(v[j], ix[j], v[i], ix[i]) : better(v[i], ix[i], v[j], ix[j]);
            if (sw) {
              const float tv = v[i];
              v[i] = v[j];
              v[j] = tv;
              const int ti = ix[i];
              ix[i] = ix[j];
              ix[j] = ti;
            }
          }
        }
      }
    }
    float sel_v = 0.f;
    int sel_i = 0;
    for (int r = 0; r < k; ++r) {
      float wv = v[0];
      int wi = ix[0];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, wi, o);
        if (better(ov, oi, wv, wi)) {
          wv = ov;
          wi = oi;
        }
      }
      if (lane == r) {
        sel_v = wv;
        sel_i = wi;
      }
      if (ix[0] == wi) {  // expert ids are unique: this lane owned the winner
#pragma unroll
        for (int i = 0; i + 1 < P; ++i) {
          v[i] = v[i + 1];
          ix[i] = ix[i + 1];
        }
        v[P - 1] = -INFINITY;
        ix[P - 1] = 0x7fffffff;
      }
    }
    // softmax over the selected logits (lane r holds slot r); the max is slot 0
    const float vmax = __shfl_sync(0xffffffffu, sel_v, 0);
    const float ex = (lane < k) ? expf(sel_v - vmax) : 0.f;
    float sum = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane < k) {
      topk_idx[(long long)t * k + lane] = sel_i;
      topk_gate[(long long)t * k + lane] = ex / sum;
      atomicAdd(&s_counts[sel_i], 1);
    }
  }
  __syncthreads();
  // expert-major layout [N][n_chunks]: the scan reads one expert's chunks contiguously
  for (int e = threadIdx.x; e < n_experts; e += blockDim.x)
    chunk_counts[(long long)e * gridDim.x + blockIdx.x] = s_counts[e];
}

// candidates per lane: the next power of two >= ceil(N / 32)
inline int topk_lane_candidates(int n_experts) {
  int p = 1;
  while (32 * p < n_experts) p <<= 1;
  return p;
}

inline cudaError_t launch_topk_hist(int n_chunks, int threads, cudaStream_t s, const float* logits, const float* bias,
                                    int T, int N, int K, int ct, int* idx, float* gate, int* chunk_counts) {
  const size_t sm = (size_t)N * sizeof(int);
  switch (topk_lane_candidates(N)) {
    case 1: topk_hist_kernel<1><<<n_chunks, threads, sm, s>>>(logits, bias, T, N, K, ct, idx, gate, chunk_counts); break;
    case 2: topk_hist_kernel<2><<<n_chunks, threads, sm, s>>>(logits, bias, T, N, K, ct, idx, gate, chunk_counts); break;
    case 4: topk_hist_kernel<4><<<n_chunks, threads, sm, s>>>(logits, bias, T, N, K, ct, idx, gate, chunk_counts); break;
    case 8: topk_hist_kernel<8><<<n_chunks, threads, sm, s>>>(logits, bias, T, N, K, ct, idx, gate, chunk_counts); break;
    case 16: topk_hist_kernel<16><<<n_chunks, threads, sm, s>>>(logits, bias, T, N, K, ct, idx, gate, chunk_counts); break;
    default: topk_hist_kernel<32><<<n_chunks, threads, sm, s>>>(logits, bias, T, N, K, ct, idx, gate, chunk_counts); break;
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Expert totals, exclusive offsets, per-chunk bases and the grouped-GEMM unit lists.
// Single block of 1024 threads; thread e owns expert e (N <= 1024).
// ------------------------------------------------------------------------------------------------
struct UnitListSpec {
  GemmUnit* units;     // output list
  int* num_units;      // output count
  int feat;            // output features per expert (rows of that expert's weight)
  int tile_tokens;     // tokens per unit (the GEMM variant's BN_MAX)
  int max_units;       // capacity
};

__device__ __forceinline__ int block_exclusive_scan(int v, int* s_tmp, int& total) {
  // s_tmp: 32 ints of shared memory; blockDim.x == 1024
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = s_tmp[lane];
    int ws = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ws, o);
      if (lane >= o) ws += y;
    }
    s_tmp[lane] = ws - w;  // exclusive prefix of warp totals
    if (lane == 31) s_tmp[32] = ws;
  }
  __syncthreads();
  const int r = s_tmp[warp] + x - v;
  total = s_tmp[32];
  __syncthreads();
  return r;
}

// Dynamic shared memory of scan_units_kernel: the [N][n_chunks] histogram with rows padded by one
// word (conflict-free per-expert walks).
inline size_t scan_smem_bytes(int n_experts, int n_chunks) { return (size_t)n_experts * (n_chunks + 1) * sizeof(int); }

__global__ void __launch_bounds__(1024)
    scan_units_kernel(const int* __restrict__ chunk_counts, int n_chunks, int n_experts, int* __restrict__ counts,
                      int* __restrict__ offsets, int* __restrict__ chunk_base, UnitListSpec l1, UnitListSpec l2,
                      int* __restrict__ tile0, unsigned* status) {
  // chunk_counts / chunk_base are expert-major: [N][n_chunks]
  extern __shared__ int s_cc[];  // [N][n_chunks + 1]
  __shared__ int s_tmp[33];
  const int pitch = n_chunks + 1;
  const int total_words = n_experts * n_chunks;
  for (int i = threadIdx.x; i < total_words; i += blockDim.x) {
    const int e = i / n_chunks, c = i - e * n_chunks;
    s_cc[e * pitch + c] = chunk_counts[i];
  }
  __syncthreads();
  const int e = threadIdx.x;
  int c_e = 0;
  if (e < n_experts)
    for (int c = 0; c < n_chunks; ++c) c_e += s_cc[e * pitch + c];
  int total;
  const int off = block_exclusive_scan(c_e, s_tmp, total);
  if (e < n_experts) {
    counts[e] = c_e;
    offsets[e] = off;
    int run = off;  // chunk bases, in place
    for (int c = 0; c < n_chunks; ++c) {
      const int v = s_cc[e * pitch + c];
      s_cc[e * pitch + c] = run;
      run += v;
    }
  }
  if (e == 0) offsets[n_experts] = total;
  __syncthreads();
  for (int i = threadIdx.x; i < total_words; i += blockDim.x) {
    const int ex = i / n_chunks, c = i - ex * n_chunks;
    chunk_base[i] = s_cc[ex * pitch + c];
  }
  // unit lists: expert-major, token block next, feature block fastest.  Consecutive threads write
  // consecutive units (16-byte stores); a unit finds its expert by binary search over the experts'
  // first-unit indices.  Token tiles are numbered expert-major: expert e owns tiles tile0[e] ...
  __shared__ int s_u0[1025];
  __shared__ int s_cnt[1024];
  __shared__ int s_offs[1024];
  __shared__ int s_t0[1024];
  const int tile_tokens = l1.units ? l1.tile_tokens : 64;
  int n_tiles;
  const int t0 = block_exclusive_scan((e < n_experts) ? (c_e + tile_tokens - 1) / tile_tokens : 0, s_tmp, n_tiles);
  if (e < n_experts) {
    s_cnt[e] = c_e;
    s_offs[e] = off;
    s_t0[e] = t0;
    if (tile0) tile0[e] = t0;
  }
  if (e == 0 && tile0) tile0[n_experts] = n_tiles;
#pragma unroll 1
  for (int li = 0; li < 2; ++li) {
    const UnitListSpec& L = li ? l2 : l1;
    if (L.units == nullptr) continue;
    const int nft = (L.feat + BLOCK_M - 1) / BLOCK_M;
    const int ntt = (c_e + L.tile_tokens - 1) / L.tile_tokens;
    const int nu = (e < n_experts) ? ntt * nft : 0;
    int nu_total;
    const int u0 = block_exclusive_scan(nu, s_tmp, nu_total);  // ends with __syncthreads
    if (e < n_experts) s_u0[e] = u0;
    if (e == 0) {
      s_u0[n_experts] = nu_total;
      *L.num_units = min(nu_total, L.max_units);
      if (nu_total > L.max_units) atomicOr(status, DEV_STATUS_BAD_INDEX);
    }
    __syncthreads();
    const int n_write = min(nu_total, L.max_units);
    for (int u = threadIdx.x; u < n_write; u += blockDim.x) {
      int lo = 0, hi = n_experts - 1;  // largest expert whose first unit is <= u
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_u0[mid] <= u) lo = mid;
        else hi = mid - 1;
      }
      const int ex = lo;
      const int local = u - s_u0[ex];
      const int tt = local / nft, ft = local - tt * nft;
      const int nv = min(L.tile_tokens, s_cnt[ex] - tt * L.tile_tokens);
      const int4 g = make_int4(ex * L.feat + ft * BLOCK_M, s_offs[ex] + tt * L.tile_tokens, ft * BLOCK_M,
                               nv | (min(BLOCK_M, L.feat - ft * BLOCK_M) << 16));
      int4* dst = reinterpret_cast<int4*>(&L.units[u]);
      dst[0] = g;
      dst[1] = make_int4(s_t0[ex] + tt, 0, 0, 0);
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------------------------
// Stable row assignment.  One warp per chunk walks the chunk's assignments in (token, slot) order,
// 32 at a time: lanes holding the same expert are ranked with __match_any_sync, and a per-expert
// running base (from scan_units_kernel) gives each assignment its grouped row.
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(32)
    assign_rows_kernel(const int* __restrict__ topk_idx, const float* __restrict__ topk_gate,
                       const int* __restrict__ chunk_base, int T, int n_experts, int k, int chunk_tokens,
                       int* __restrict__ row_of, int* __restrict__ tok_of_row, float* __restrict__ gate_of_row,
                       unsigned* status) {
  extern __shared__ int s_base[];  // [n_experts]
  const int lane = threadIdx.x;
  for (int e = lane; e < n_experts; e += 32) s_base[e] = chunk_base[(long long)e * gridDim.x + blockIdx.x];
  __syncwarp();
  const int t_begin = blockIdx.x * chunk_tokens;
  const int t_end = min(T, t_begin + chunk_tokens);
  const long long a_begin = (long long)t_begin * k, a_end = (long long)t_end * k;
  const long long TK = (long long)T * k;
  for (long long a0 = a_begin; a0 < a_end; a0 += 32) {
    const long long a = a0 + lane;
    const bool act = a < a_end;
    int e = act ? topk_idx[a] : -1 - lane;  // inactive lanes get unique keys
    const bool e_ok = e >= 0 && e < n_experts;
    if (act && !e_ok) atomicOr(status, DEV_STATUS_BAD_INDEX);
    const float g = act ? topk_gate[a] : 0.f;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int leader = __ffs(peers) - 1;
    int base = 0;
    if (act && e_ok) base = s_base[e];
    __syncwarp();
    if (act && e_ok && lane == leader) s_base[e] = base + __popc(peers);
    __syncwarp();
    if (act) {
      const int row = e_ok ? base + rank : -1;
      if (row >= 0 && row < TK) {
        row_of[a] = row;
        tok_of_row[row] = (int)(a / k);
        gate_of_row[row] = g;
      } else {
        if (e_ok) atomicOr(status, DEV_STATUS_BAD_INDEX);
        row_of[a] = -1;
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------
// Gather of latent rows into expert-grouped order: h_perm[r] = h[tok_of_row[r]].  Grid-stride over
// groups of 8 grouped rows per warp, so each lane keeps 8 independent 16-byte loads in flight.
// ------------------------------------------------------------------------------------------------
constexpr int GATHER_ROWS = 8;

__global__ void __launch_bounds__(256)
    gather_rows_kernel(const __nv_bfloat16* __restrict__ h, const int* __restrict__ tok_of_row, long long n_rows,
                       int T, int latent, __nv_bfloat16* __restrict__ h_perm, unsigned* status) {
  const int lane = threadIdx.x & 31;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int vpr = latent / 8;
  for (long long r0 = warp * GATHER_ROWS; r0 < n_rows; r0 += nwarps * GATHER_ROWS) {
    int tok[GATHER_ROWS];
#pragma unroll
    for (int j = 0; j < GATHER_ROWS; ++j) {
      const long long r = r0 + j;
      int t = (r < n_rows) ? tok_of_row[r] : -1;
      if (r < n_rows && (t < 0 || t >= T)) {
        if (lane == 0) atomicOr(status, DEV_STATUS_BAD_INDEX);
        t = -1;
      }
      tok[j] = t;
    }
    for (int i = lane; i < vpr; i += 32) {
      uint4 buf[GATHER_ROWS];
#pragma unroll
      for (int j = 0; j < GATHER_ROWS; ++j)
        if (tok[j] >= 0) buf[j] = reinterpret_cast<const uint4*>(h + (long long)tok[j] * latent)[i];
#pragma unroll
      for (int j = 0; j < GATHER_ROWS; ++j)
        if (tok[j] >= 0) reinterpret_cast<uint4*>(h_perm + (r0 + j) * latent)[i] = buf[j];
    }
  }
}

// ------------------------------------------------------------------------------------------------
// combine: zu[t, 0:latent] = bf16( sum_k o[row_of[t, k], :] (+ add[t, :]) ), slot order, fp32
// accumulation; the fp32 addend (a standard MoE's shared-expert output) is added last
// ------------------------------------------------------------------------------------------------
__global__ void combine_kernel(const __nv_bfloat16* __restrict__ o, const int* __restrict__ row_of, int T, int k,
                               int latent, __nv_bfloat16* __restrict__ zu, long long ld_zu, long long n_rows,
                               unsigned* status, const float* __restrict__ add = nullptr, long long ld_add = 0) {
  const int vpr = latent / 8;  // 8 bf16 per thread
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long t = gid / vpr;
  const int v = (int)(gid % vpr);
  if (t >= T) return;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < k; ++s) {
    const int row = row_of[t * k + s];
    if (row < 0 || row >= n_rows) {
      atomicOr(status, DEV_STATUS_BAD_INDEX);
      continue;
    }
    const uint4 q = *reinterpret_cast<const uint4*>(o + (long long)row * latent + v * 8);
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(p[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
  if (add != nullptr) {
    const float4* pa = reinterpret_cast<const float4*>(add + t * ld_add + v * 8);
    const float4 a0 = pa[0], a1 = pa[1];
    acc[0] += a0.x;
    acc[1] += a0.y;
    acc[2] += a0.z;
    acc[3] += a0.w;
    acc[4] += a1.x;
    acc[5] += a1.y;
    acc[6] += a1.z;
    acc[7] += a1.w;
  }
  uint4 out;
  __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
  for (int i = 0; i < 4; ++i) po[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
  *reinterpret_cast<uint4*>(zu + t * ld_zu + v * 8) = out;
}

// ------------------------------------------------------------------------------------------------
// weight preparation: copy or convert a [rows, cols] matrix (bf16 or fp32 source) into a bf16
// destination with its own row pitch and column offset (used to stack/concatenate weights).
// ------------------------------------------------------------------------------------------------
__global__ void convert_2d_kernel(const void* __restrict__ src, int src_is_f32, long long rows, int cols,
                                  long long src_ld, __nv_bfloat16* __restrict__ dst, long long dst_ld, int dst_col0) {
  const long long total = rows * cols;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / cols;
    const int c = (int)(i % cols);
    __nv_bfloat16 v;
    if (src_is_f32)
      v = __float2bfloat16_rn(reinterpret_cast<const float*>(src)[r * src_ld + c]);
    else
      v = reinterpret_cast<const __nv_bfloat16*>(src)[r * src_ld + c];
    dst[r * dst_ld + dst_col0 + c] = v;
  }
}

}  // namespace lmoe
