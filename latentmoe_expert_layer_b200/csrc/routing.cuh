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

#include <utility>

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
// top-K + softmax + per-chunk expert histogram.  A chunk of `chunk_tokens` consecutive tokens is
// handled by `parts` blocks, one warp per token.  Lane j holds the candidates j, j + 32, ... (P of
// them) as order-preserving 32-bit keys.  The K-th largest key X is built two bits at a time from
// warp-wide counts; the selection is every key above X plus the lowest expert indices among the keys
// equal to X (ranked with ballots in index order); a warp bitonic sort puts the K selections in
// output order (value desc, index asc).  Requires K <= 32 and N <= 32 * P.
// ------------------------------------------------------------------------------------------------

// One token's top-K on one warp: val[i] is logit e = 32 i + lane (bias not included; the caller
// loads every candidate first, so that all its loads are in flight together).  Writes the K expert
// ids and softmax gates of the token (slot r at out_idx[r], out_gate[r]) and counts the selections
// into the shared-memory histogram s_counts.  s_key / s_idx: 32 words each of warp-private scratch.
template <int P>
__device__ __forceinline__ void topk_one_token(const float (&val)[P], const float* __restrict__ bias, int n_experts,
                                               int k, uint32_t* s_key, int* s_idx, int* __restrict__ out_idx,
                                               float* __restrict__ out_gate, int* s_counts) {
  const int lane = threadIdx.x & 31;
  // order-preserving keys: a larger logit has a larger key, -0 and +0 share one; padding is 0
  uint32_t key[P];
#pragma unroll
  for (int i = 0; i < P; ++i) {
    const int e = i * 32 + lane;
    if (e < n_experts) {
      const uint32_t u = __float_as_uint(__fadd_rn(val[i] + (bias ? bias[e] : 0.f), 0.f));
      key[i] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    } else {
      key[i] = 0u;
    }
  }
  // the K-th largest key X: the largest value with at least K keys >= X, built two bits at a
  // time (three independent warp-wide counts per step)
  uint32_t X = 0u;
#pragma unroll 1
  for (int b = 30; b >= 0; b -= 2) {
    const uint32_t Y1 = X | (1u << b), Y2 = X | (2u << b), Y3 = X | (3u << b);
    int c1 = 0, c2 = 0, c3 = 0;
#pragma unroll
    for (int i = 0; i < P; ++i) {
      c1 += key[i] >= Y1;
      c2 += key[i] >= Y2;
      c3 += key[i] >= Y3;
    }
    c1 = __reduce_add_sync(0xffffffffu, c1);
    c2 = __reduce_add_sync(0xffffffffu, c2);
    c3 = __reduce_add_sync(0xffffffffu, c3);
    X = c3 >= k ? Y3 : c2 >= k ? Y2 : c1 >= k ? Y1 : X;
  }
  // selected: every key above X, then the lowest expert indices among the keys equal to X
  int above = 0;
#pragma unroll
  for (int i = 0; i < P; ++i) above += key[i] > X;
  const int need = k - __reduce_add_sync(0xffffffffu, above);
  const unsigned lt = (1u << lane) - 1u;
  int tie_base = 0, pos_base = 0;
#pragma unroll
  for (int i = 0; i < P; ++i) {
    const unsigned tie = __ballot_sync(0xffffffffu, key[i] == X);
    const bool sel = key[i] > X || (key[i] == X && tie_base + __popc(tie & lt) < need);
    tie_base += __popc(tie);
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int pos = pos_base + __popc(sb & lt);
      s_key[pos] = key[i];
      s_idx[pos] = i * 32 + lane;
    }
    pos_base += __popc(sb);
  }
  __syncwarp();
  uint32_t mk = lane < k ? s_key[lane] : 0u;
  int mi = lane < k ? s_idx[lane] : 0x7fffffff;
  __syncwarp();
  // bitonic sort of the K selections over the warp: key descending, then index ascending
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint32_t ok = __shfl_xor_sync(0xffffffffu, mk, stride);
      const int oi = __shfl_xor_sync(0xffffffffu, mi, stride);
      const bool other_better = ok > mk || (ok == mk && oi < mi);
      const bool keep_better = ((lane & stride) == 0) == ((lane & size) == 0);
      if (keep_better == other_better) {
        mk = ok;
        mi = oi;
      }
    }
  }
  const uint32_t ub = (mk & 0x80000000u) ? (mk & 0x7fffffffu) : ~mk;
  const float sel_v = __uint_as_float(ub);
  // softmax over the selected logits (lane r holds slot r); the max is slot 0
  const float vmax = __shfl_sync(0xffffffffu, sel_v, 0);
  const float ex = (lane < k) ? expf(sel_v - vmax) : 0.f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    out_idx[lane] = mi;
    out_gate[lane] = ex / sum;
    atomicAdd(&s_counts[mi], 1);
  }
}

template <int P>
__global__ void __launch_bounds__(1024)
    topk_hist_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T, int n_experts,
                     int k, int chunk_tokens, int parts, int* __restrict__ topk_idx, float* __restrict__ topk_gate,
                     int* __restrict__ chunk_counts) {
  extern __shared__ int s_counts[];  // [n_experts], then per warp 32 keys + 32 indices
  for (int e = threadIdx.x; e < n_experts; e += blockDim.x) s_counts[e] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  // `parts` blocks share a chunk: block b takes part (b mod parts) of chunk (b / parts)
  const int chunk = blockIdx.x / parts, part = blockIdx.x - chunk * parts;
  const int n_chunks = gridDim.x / parts;
  const int sub = (chunk_tokens + parts - 1) / parts;
  const int t_begin = chunk * chunk_tokens + part * sub;
  const int t_end = min(min(T, (chunk + 1) * chunk_tokens), t_begin + sub);
  uint32_t* s_key = reinterpret_cast<uint32_t*>(s_counts + n_experts) + warp * 64;
  int* s_idx = reinterpret_cast<int*>(s_key + 32);
  for (int t = t_begin + warp; t < t_end; t += nwarps) {
    const float* lrow = logits + (long long)t * n_experts;
    float val[P];
#pragma unroll
    for (int i = 0; i < P; ++i) val[i] = (i * 32 + lane < n_experts) ? lrow[i * 32 + lane] : 0.f;
    topk_one_token<P>(val, bias, n_experts, k, s_key, s_idx, topk_idx + (long long)t * k, topk_gate + (long long)t * k,
                      s_counts);
  }
  __syncthreads();
  // expert-major layout [N][n_chunks]: the scan reads one expert's chunks contiguously; blocks that
  // share a chunk add into a zeroed histogram
  for (int e = threadIdx.x; e < n_experts; e += blockDim.x) {
    int* dst = chunk_counts + (long long)e * n_chunks + chunk;
    if (parts == 1) *dst = s_counts[e];
    else if (s_counts[e]) atomicAdd(dst, s_counts[e]);
  }
}

// candidates per lane: the next power of two >= ceil(N / 32)
inline int topk_lane_candidates(int n_experts) {
  int p = 1;
  while (32 * p < n_experts) p <<= 1;
  return p;
}

// parts > 1: blocks per chunk (the caller zeroes chunk_counts first); threads per block from the
// tokens each block takes
inline cudaError_t launch_topk_hist(int n_chunks, int parts, cudaStream_t s, const float* logits, const float* bias,
                                    int T, int N, int K, int ct, int* idx, float* gate, int* chunk_counts) {
  const int sub = (ct + parts - 1) / parts;
  const int threads = 32 * (sub < 32 ? sub : 32);
  const size_t sm = (size_t)N * sizeof(int) + (size_t)(threads / 32) * 64 * sizeof(int);
  const int grid = n_chunks * parts;
#define LMOE_TOPK(PP) \
  topk_hist_kernel<PP><<<grid, threads, sm, s>>>(logits, bias, T, N, K, ct, parts, idx, gate, chunk_counts)
  switch (topk_lane_candidates(N)) {
    case 1: LMOE_TOPK(1); break;
    case 2: LMOE_TOPK(2); break;
    case 4: LMOE_TOPK(4); break;
    case 8: LMOE_TOPK(8); break;
    case 16: LMOE_TOPK(16); break;
    default: LMOE_TOPK(32); break;
  }
#undef LMOE_TOPK
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Expert totals, exclusive offsets, per-chunk bases, first token tiles and each expert's first unit
// in the two grouped-GEMM unit lists (build_units_kernel then writes the lists over the whole grid).
// Single block of 1024 threads; thread e owns expert e (N <= 1024).
// ------------------------------------------------------------------------------------------------
struct UnitListSpec {
  GemmUnit* units;     // output list
  int* num_units;      // output count
  int feat;            // output features per expert (rows of that expert's weight)
  int tile_tokens;     // tokens per unit (the GEMM variant's BN_MAX)
  int max_units;       // capacity
  int* u0;             // [N + 1] first unit of each expert, then the total (written by the scan)
  int tile_rows;       // weight rows per unit: 128, or 256 for the CTA-pair variant
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
  // 8 loads in flight per thread at a time (a plain loop waits for each before the next)
  for (int i0 = threadIdx.x; i0 < total_words; i0 += 8 * blockDim.x) {
    int vals[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = i0 + j * blockDim.x;
      vals[j] = i < total_words ? chunk_counts[i] : 0;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = i0 + j * blockDim.x;
      if (i < total_words) {
        const int e = i / n_chunks, c = i - e * n_chunks;
        s_cc[e * pitch + c] = vals[j];
      }
    }
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
  // unit lists (written by build_units_kernel): expert-major, token block next, feature block
  // fastest; here only each expert's first unit.  Token tiles are numbered expert-major: expert e
  // owns tiles tile0[e] ...
  const int tile_tokens = l1.units ? l1.tile_tokens : 64;
  int n_tiles;
  const int t0 = block_exclusive_scan((e < n_experts) ? (c_e + tile_tokens - 1) / tile_tokens : 0, s_tmp, n_tiles);
  if (e < n_experts && tile0) tile0[e] = t0;
  if (e == 0 && tile0) tile0[n_experts] = n_tiles;
#pragma unroll 1
  for (int li = 0; li < 2; ++li) {
    const UnitListSpec& L = li ? l2 : l1;
    if (L.units == nullptr) continue;
    const int nft = (L.feat + L.tile_rows - 1) / L.tile_rows;
    const int ntt = (c_e + L.tile_tokens - 1) / L.tile_tokens;
    const int nu = (e < n_experts) ? ntt * nft : 0;
    int nu_total;
    const int u0 = block_exclusive_scan(nu, s_tmp, nu_total);  // ends with __syncthreads
    if (e < n_experts) L.u0[e] = u0;
    if (e == 0) {
      L.u0[n_experts] = nu_total;
      *L.num_units = min(nu_total, L.max_units);
      if (nu_total > L.max_units) atomicOr(status, DEV_STATUS_BAD_INDEX);
    }
  }
}

// ------------------------------------------------------------------------------------------------
// Grouped-GEMM unit lists from the scan's per-expert first units, one unit per thread over the
// whole grid: a unit finds its expert by binary search over the first-unit indices (the largest
// expert whose first unit is <= u, which skips experts without units).
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    build_units_kernel(const int* __restrict__ counts, const int* __restrict__ offsets,
                       const int* __restrict__ tile0, int n_experts, UnitListSpec l1, UnitListSpec l2) {
  const int n1 = l1.units ? *l1.num_units : 0;
  const int n2 = l2.units ? *l2.num_units : 0;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n1 + n2; i += stride) {
    const bool second = i >= n1;
    const UnitListSpec& L = second ? l2 : l1;
    const int u = (int)(second ? i - n1 : i);
    int lo = 0, hi = n_experts - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(L.u0 + mid) <= u) lo = mid;
      else hi = mid - 1;
    }
    const int ex = lo;
    const int nft = (L.feat + L.tile_rows - 1) / L.tile_rows;
    const int local = u - __ldg(L.u0 + ex);
    const int tt = local / nft, ft = local - tt * nft;
    const int nv = min(L.tile_tokens, __ldg(counts + ex) - tt * L.tile_tokens);
    const int4 g = make_int4(ex * L.feat + ft * L.tile_rows, __ldg(offsets + ex) + tt * L.tile_tokens,
                             ft * L.tile_rows, nv | (min(L.tile_rows, L.feat - ft * L.tile_rows) << 16));
    int4* dst = reinterpret_cast<int4*>(&L.units[u]);
    dst[0] = g;
    dst[1] = make_int4(__ldg(tile0 + ex) + tt, 0, 0, 0);
  }
}

// ------------------------------------------------------------------------------------------------
// Stable row assignment.  One block per chunk; its W warps take contiguous parts of the chunk's
// assignments in (token, slot) order.  Each warp counts its part per expert, the per-warp bases
// follow from the chunk's per-expert base (scan_units_kernel) and the earlier warps' counts, and then
// each warp walks its part 32 at a time: lanes holding the same expert are ranked with
// __match_any_sync on top of the warp's running base.  W = 1 (32 threads) works as well.
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    assign_rows_kernel(const int* __restrict__ topk_idx, const float* __restrict__ topk_gate,
                       const int* __restrict__ chunk_base, int T, int n_experts, int k, int chunk_tokens,
                       int* __restrict__ row_of, int* __restrict__ tok_of_row, float* __restrict__ gate_of_row,
                       unsigned* status) {
  extern __shared__ int s_hist[];  // [W][n_experts]: per warp, then per-warp running bases
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, W = blockDim.x >> 5;
  for (int i = threadIdx.x; i < W * n_experts; i += blockDim.x) s_hist[i] = 0;
  const int t_begin = blockIdx.x * chunk_tokens;
  const int t_end = min(T, t_begin + chunk_tokens);
  const long long a_begin = (long long)t_begin * k, a_end = (long long)t_end * k;
  const long long TK = (long long)T * k;
  // warp w walks the w-th contiguous sub-range of the chunk's assignments, in (token, slot) order
  const long long per = (a_end - a_begin + W - 1) / W;
  const long long s_begin = min(a_end, a_begin + warp * per), s_end = min(a_end, s_begin + per);
  int* my = s_hist + warp * n_experts;
  __syncthreads();
  // 1. per-warp expert counts (the leader of each group of equal experts adds the group's size)
  for (long long a0 = s_begin; a0 < s_end; a0 += 32) {
    const long long a = a0 + lane;
    const int e = a < s_end ? topk_idx[a] : -1 - lane;
    const bool e_ok = e >= 0 && e < n_experts;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e_ok && lane == __ffs(peers) - 1) my[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // 2. per-warp bases: the chunk's base for the expert plus the counts of the earlier warps
  for (int e = threadIdx.x; e < n_experts; e += blockDim.x) {
    int run = chunk_base[(long long)e * gridDim.x + blockIdx.x];
    for (int w = 0; w < W; ++w) {
      const int v = s_hist[w * n_experts + e];
      s_hist[w * n_experts + e] = run;
      run += v;
    }
  }
  __syncthreads();
  // 3. ranks: lanes holding the same expert are ranked with __match_any_sync on top of the warp's
  //    running base; the next round's ids and gates load while this round is ranked
  int e_next = (s_begin + lane < s_end) ? topk_idx[s_begin + lane] : 0;
  float g_next = (s_begin + lane < s_end) ? topk_gate[s_begin + lane] : 0.f;
  for (long long a0 = s_begin; a0 < s_end; a0 += 32) {
    const long long a = a0 + lane;
    const bool act = a < s_end;
    const int e = act ? e_next : -1 - lane;  // inactive lanes get unique keys
    const float g = act ? g_next : 0.f;
    if (a + 32 < s_end) {
      e_next = topk_idx[a + 32];
      g_next = topk_gate[a + 32];
    }
    const bool e_ok = e >= 0 && e < n_experts;
    if (act && !e_ok) atomicOr(status, DEV_STATUS_BAD_INDEX);
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int leader = __ffs(peers) - 1;
    int base = 0;
    if (act && e_ok) base = my[e];
    __syncwarp();
    if (act && e_ok && lane == leader) my[e] = base + __popc(peers);
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
// BATCH: every row index, then the rows 8 at a time, are in flight together (k <= 32): few memory
// latencies per token, for small grids that cannot hide latency with many threads; otherwise one row
// at a time with fewer registers, for occupancy.  Both sum in slot order.
template <bool BATCH>
__global__ void combine_kernel(const __nv_bfloat16* __restrict__ o, const int* __restrict__ row_of, int T, int k,
                               int latent, __nv_bfloat16* __restrict__ zu, long long ld_zu, long long n_rows,
                               unsigned* status, const float* __restrict__ add, long long ld_add) {
  griddep_launch_dependents();
  griddep_wait();  // o comes from the launch before
  const int vpr = latent / 8;  // 8 bf16 per thread
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long t = gid / vpr;
  const int v = (int)(gid % vpr);
  if (t >= T) return;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  auto add_row = [&](const uint4& q) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(p[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  };
  if constexpr (!BATCH) {
    for (int s = 0; s < k; ++s) {
      const int row = row_of[t * k + s];
      if (row < 0 || row >= n_rows) {
        atomicOr(status, DEV_STATUS_BAD_INDEX);
        continue;
      }
      add_row(*reinterpret_cast<const uint4*>(o + (long long)row * latent + v * 8));
    }
  } else {
  int rows[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) rows[j] = j < k ? row_of[t * k + j] : -1;
#pragma unroll
  for (int s0 = 0; s0 < 32; s0 += 8) {
    if (s0 >= k) break;
    uint4 q[8];
    bool okq[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int row = rows[s0 + j];
      okq[j] = s0 + j < k && row >= 0 && row < n_rows;
      if (s0 + j < k && !okq[j]) atomicOr(status, DEV_STATUS_BAD_INDEX);
      if (okq[j]) q[j] = *reinterpret_cast<const uint4*>(o + (long long)row * latent + v * 8);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (okq[j]) add_row(q[j]);
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
// Sum of a split-K router GEMM's slices (fixed slice order): part[s] is [T, n_logits + n_h] fp32;
// columns < n_logits go to the fp32 logits, the rest to bf16 h.  One thread per 4 columns
// (n_logits is a multiple of 16, so a group never straddles the two outputs).
__global__ void __launch_bounds__(256)
    split_reduce_kernel(const float* __restrict__ part, int n_slices, long long slice_stride, int T, int n_logits,
                        int n_h, float* __restrict__ logits, __nv_bfloat16* __restrict__ h) {
  const int W = n_logits + n_h;
  const int vpr = W / 4;
  const long long total = (long long)T * vpr;
  for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < total;
       g += (long long)gridDim.x * blockDim.x) {
    const long long t = g / vpr;
    const int col = (int)(g - t * vpr) * 4;
    const float* src = part + t * W + col;
    float4 a = *reinterpret_cast<const float4*>(src);
    for (int sl = 1; sl < n_slices; ++sl) {
      const float4 b = *reinterpret_cast<const float4*>(src + sl * slice_stride);
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    if (col < n_logits) {
      *reinterpret_cast<float4*>(logits + t * n_logits + col) = a;
    } else {
      __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(h + t * n_h + (col - n_logits)) = pk;
    }
  }
}

// combine over T tokens of `latent` columns: the batched variant while the grid is below ~8 warps
// per SM
// Launch with programmatic stream serialisation (the kernel calls griddep_wait before it reads what
// the previous launch wrote): its launch and set-up overlap the previous kernel's tail.
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*kernel)(P...), int grid, int threads, size_t smem, cudaStream_t s, int cluster,
                       A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cluster > 1) {  // clusters of `cluster` consecutive CTAs (grid is a multiple of it)
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

inline cudaError_t launch_combine(int num_sms, cudaStream_t s, const __nv_bfloat16* o, const int* row_of, int T,
                                  int k, int latent, __nv_bfloat16* out, long long ld_out, long long n_rows,
                                  unsigned* status, const float* add = nullptr, long long ld_add = 0) {
  const long long threads = (long long)T * (latent / 8);
  const int blocks = (int)((threads + 255) / 256);
  if (threads <= (long long)num_sms * 256)
    return launch_pdl(combine_kernel<true>, blocks, 256, 0, s, 1, o, row_of, T, k, latent, out, ld_out, n_rows, status,
                      add, ld_add);
  return launch_pdl(combine_kernel<false>, blocks, 256, 0, s, 1, o, row_of, T, k, latent, out, ld_out, n_rows, status,
                    add, ld_add);
}

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
