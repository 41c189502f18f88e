// Decode-sized routing in ONE cooperative launch: router slice sum, top-K + gates, expert histogram,
// expert offsets, grouped-GEMM unit lists, stable row assignment and the gather of latent rows.
//
// At decode sizes (a few hundred tokens) every one of these steps is latency-bound, and as separate
// kernels they cost a launch gap each.  The grid has one block per SM; the first n_chunks blocks
// ("chunk blocks") each own a chunk of chunk_tokens consecutive tokens:
//
//   phase 1  chunk blocks, one warp per token: logits = sum of the router GEMM's K-slice partials
//            (fixed slice order), top-K and softmax gates (topk_one_token), the chunk's expert
//            histogram -> chunk_counts[b][e]; all blocks: h = bf16(sum of the W_down slices)
//   -------  grid barrier
//   phase 2  chunk blocks, redundantly: per-expert totals over the chunks and the block's own
//            prefix, exclusive scans (expert offsets, first token tiles, first units of the two unit
//            lists); block 0 publishes them; the unit lists are written by all chunk blocks; block b
//            assigns the grouped rows of its chunk's (token, slot) pairs (stable in (token, slot)
//            order)
//   -------  grid barrier
//   phase 3  all blocks: the gather h_perm[r] = h[tok_of_row[r]]
//
// NVFP4 experts (fp4 != 0): phase 1 also takes max |x| and max |h| (of the bf16 h) over the grid;
// in phase 2 the blocks without a chunk quantise x (the shared expert's input, in the expert
// launch's dense tile atoms) and h once per token with the dynamic tensor scales; phase 3 copies
// each grouped row's h codes and scales (tile-local atoms) instead of gathering bf16 rows.
//
// The grid barrier is self-resetting (an arrival count and a generation word, both zero when the
// layer is created) and its wait is bounded by wall-clock time: on expiry the block raises
// DEV_STATUS_TIMEOUT and returns (the host then resets the barrier words when it reads the status).
// The launch is cooperative, so all blocks are resident together.
#pragma once
#include <cuda_bf16.h>

#include "nvfp4.cuh"
#include "ptx.cuh"
#include "routing.cuh"

namespace lmoe {

struct RouteFusedArgs {
  const float* part;           // router K-slice partials [ks][T][N + l] (logit columns first)
  int ks;
  long long slice_stride;      // elements between slices (T * (N + l))
  const float* bias;           // [N] or nullptr
  int T, N, K, l;
  int chunk_tokens;            // tokens per chunk block
  int n_chunks;                // chunk blocks: ceil(T / chunk_tokens) <= gridDim.x
  float* logits;               // [T, N] out
  __nv_bfloat16* h;            // [T, l] out
  int* idx;                    // [T, K] out
  float* gate;                 // [T, K] out
  int* chunk_counts;           // [n_chunks][N] scratch
  int* counts;                 // [N] out
  int* offsets;                // [N + 1] out
  int* tile0;                  // [N + 1] out: first token tile of each expert, then the total
  UnitListSpec l1, l2;         // grouped-GEMM unit lists (u0 / num_units written here)
  int* row_of;                 // [T * K] out
  int* tok_of_row;             // [T * K] out
  float* gate_of_row;          // [T * K] out
  __nv_bfloat16* h_perm;       // [T * K, l] out: grouped latent rows
  int* zero_words;             // words zeroed for the launches that follow (their unit counters)
  int n_zero;
  unsigned* bar;               // [2]: grid-barrier arrival count, generation
  unsigned* status;
  unsigned long long timeout_ns;
  // NVFP4 experts
  int fp4;
  const __nv_bfloat16* x;      // [T, d] layer input
  int d;
  unsigned* amax;              // [2]: max |x|, max |h| as float bits (zero at launch)
  float* act_g;                // [2] out: tensor scales g_x, g_h
  uint8_t* xq;                 // [T, d / 2] x codes
  uint8_t* x_sf;               //   x block scales, dense tile-local atoms
  uint8_t* hq_tok;             // [T, l / 2] h codes per token
  uint8_t* h_sf_tok;           // [T, l / 16] h block scales per token (plain)
  uint8_t* hq;                 // [T * K, l / 2] grouped h codes
  uint8_t* h_sf;               //   grouped h block scales, tile-local atoms
  int tile_tokens4;            // token tile of the FP4 expert variant
  int nra4;                    // its 128-row scale atoms per tile
};

// Grid-wide barrier of a cooperative launch (every block resident).  Returns false, with
// DEV_STATUS_TIMEOUT raised, when the wait runs past limit_ns.
__device__ __forceinline__ bool grid_barrier_bounded(unsigned* bar, unsigned long long limit_ns, unsigned* status) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile unsigned* gen = bar + 1;
    const unsigned g0 = *gen;
    __threadfence();                                 // this block's writes before its arrival
    const unsigned arrived = atomicAdd(bar, 1u);
    int ok = 1;
    if (arrived == gridDim.x - 1) {
      bar[0] = 0u;                                   // reset for the next use, then release
      __threadfence();
      atomicAdd(bar + 1, 1u);
    } else {
      const uint64_t t0 = global_timer_ns();
      while (*gen == g0) {
        if (global_timer_ns() - t0 > limit_ns) {
          atomicOr(status, DEV_STATUS_TIMEOUT);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();                                 // the other blocks' writes before our reads
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// In-place exclusive scans of four arrays v0..v3 [0, n) in shared memory in one pass (one set of
// block barriers for all four); totals to tot[0..3].  s_warp: 4 x 33 ints of shared memory.
__device__ __forceinline__ void block_scan_excl4(int* v0, int* v1, int* v2, int* v3, int n, int* s_warp,
                                                 int (&tot)[4]) {
  int* v[4] = {v0, v1, v2, v3};
  const int nt = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
  const int per = (n + nt - 1) / nt;
  const int b = min(n, tid * per), e = min(n, b + per);
  int sum[4], x[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    sum[q] = 0;
    for (int i = b; i < e; ++i) sum[q] += v[q][i];
    x[q] = sum[q];
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int y = __shfl_up_sync(0xffffffffu, x[q], o);
      if (lane >= o) x[q] += y;
    }
  }
  if (lane == 31)
#pragma unroll
    for (int q = 0; q < 4; ++q) s_warp[q * 33 + warp] = x[q];
  __syncthreads();
  if (warp < 4) {  // warp q scans the warp totals of array q
    const int w = lane < nw ? s_warp[warp * 33 + lane] : 0;
    int ws = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ws, o);
      if (lane >= o) ws += y;
    }
    if (lane < nw) s_warp[warp * 33 + lane] = ws - w;
    if (lane == 31) s_warp[warp * 33 + 32] = ws;
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    int run = s_warp[q * 33 + warp] + x[q] - sum[q];
    for (int i = b; i < e; ++i) {
      const int t = v[q][i];
      v[q][i] = run;
      run += t;
    }
    tot[q] = s_warp[q * 33 + 32];
  }
  __syncthreads();
}

// Dynamic shared memory of route_fused_kernel for N experts and W warps.
inline size_t route_fused_smem(int n_experts, int warps) {
  const size_t phase1 = (size_t)n_experts * 4 + (size_t)warps * 64 * 4;
  const size_t phase2 = (size_t)5 * (n_experts + 1) * 4 + (size_t)warps * n_experts * 4;
  return phase1 > phase2 ? phase1 : phase2;
}

template <int P>
__global__ void __launch_bounds__(256) route_fused_kernel(const RouteFusedArgs a) {
  extern __shared__ int smem_i[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, W = blockDim.x >> 5;
  const int b = blockIdx.x, G = gridDim.x, nch = a.n_chunks;
  const int N = a.N, K = a.K, l = a.l, rows_w = N + l;
  const bool chunk_block = b < nch;
  const int t_begin = b * a.chunk_tokens, t_end = min(a.T, t_begin + a.chunk_tokens);

  // ------------------------------------------------------------------ phase 1
  int* s_counts = smem_i;  // [N]
  for (int e = tid; e < N; e += blockDim.x) s_counts[e] = 0;
  if (b == 0)
    for (int i = tid; i < a.n_zero; i += blockDim.x) a.zero_words[i] = 0;
  __syncthreads();
  if (chunk_block) {
    uint32_t* s_key = reinterpret_cast<uint32_t*>(s_counts + N) + warp * 64;
    int* s_idx = reinterpret_cast<int*>(s_key + 32);
    for (int t = t_begin + warp; t < t_end; t += W) {
      const float* p0 = a.part + (long long)t * rows_w;
      float* lrow = a.logits + (long long)t * N;
      // the token's logits: slice sums in slice order (every candidate's loads of one slice in
      // flight together), kept for inspection
      float val[P];
#pragma unroll
      for (int i = 0; i < P; ++i) val[i] = (i * 32 + lane < N) ? p0[i * 32 + lane] : 0.f;
      for (int s = 1; s < a.ks; ++s) {
        float w[P];
#pragma unroll
        for (int i = 0; i < P; ++i) w[i] = (i * 32 + lane < N) ? p0[s * a.slice_stride + i * 32 + lane] : 0.f;
#pragma unroll
        for (int i = 0; i < P; ++i) val[i] += w[i];
      }
#pragma unroll
      for (int i = 0; i < P; ++i)
        if (i * 32 + lane < N) lrow[i * 32 + lane] = val[i];
      topk_one_token<P>(val, a.bias, N, K, s_key, s_idx, a.idx + (long long)t * K, a.gate + (long long)t * K,
                        s_counts);
    }
  }
  // latent rows of all tokens, over the whole grid: h = bf16(sum of the W_down slices), 4 columns
  // per thread
  float amax_h = 0.f;  // NVFP4: max |h| of this thread's bf16 values
  {
    const int vpr = l / 4;
    const long long n = (long long)a.T * vpr;
    for (long long i = (long long)b * blockDim.x + tid; i < n; i += (long long)G * blockDim.x) {
      const long long t = i / vpr;
      const int col = (int)(i - t * vpr) * 4;
      const float* src = a.part + t * rows_w + N + col;
      float4 v = *reinterpret_cast<const float4*>(src);
      for (int s = 1; s < a.ks; ++s) {
        const float4 w = *reinterpret_cast<const float4*>(src + s * a.slice_stride);
        v.x += w.x;
        v.y += w.y;
        v.z += w.z;
        v.w += w.w;
      }
      __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(a.h + t * l + col) = pk;
      if (a.fp4) {
        const float2 fl = __bfloat1622float2(lo), fh = __bfloat1622float2(hi);
        amax_h = fmaxf(amax_h, fmaxf(fmaxf(fabsf(fl.x), fabsf(fl.y)), fmaxf(fabsf(fh.x), fabsf(fh.y))));
      }
    }
  }
  if (a.fp4) {
    // max |x| over the grid (8 bf16 per load), then one atomic per warp for each maximum
    float amax_x = 0.f;
    const long long n8 = (long long)a.T * a.d / 8;
    for (long long i = (long long)b * blockDim.x + tid; i < n8; i += (long long)G * blockDim.x) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(a.x) + i);
      const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(p2[j]);
        amax_x = fmaxf(amax_x, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      amax_x = fmaxf(amax_x, __shfl_xor_sync(0xffffffffu, amax_x, o));
      amax_h = fmaxf(amax_h, __shfl_xor_sync(0xffffffffu, amax_h, o));
    }
    if (lane == 0) {
      if (amax_x > 0.f) atomicMax(a.amax, __float_as_uint(amax_x));
      if (amax_h > 0.f) atomicMax(a.amax + 1, __float_as_uint(amax_h));
    }
  }
  __syncthreads();
  if (chunk_block)
    for (int e = tid; e < N; e += blockDim.x) a.chunk_counts[(long long)b * N + e] = s_counts[e];

  if (!grid_barrier_bounded(a.bar, a.timeout_ns, a.status)) return;

  // ------------------------------------------------------------------ phase 2
  if (chunk_block) {
    int* s_off = smem_i;                 // [N + 1] expert offsets
    int* s_base = s_off + (N + 1);       // [N + 1] this chunk's first row per expert
    int* s_t0 = s_base + (N + 1);        // [N + 1] first token tile per expert
    int* s_u1 = s_t0 + (N + 1);          // [N + 1] first unit per expert, list 1
    int* s_u2 = s_u1 + (N + 1);          // [N + 1] first unit per expert, list 2
    int* s_hist = s_u2 + (N + 1);        // [W][N] per-warp counts, then per-warp running bases
    __shared__ int s_warp[4 * 33];
    const int tile = a.l1.tile_tokens;
    const int nft1 = (a.l1.feat + a.l1.tile_rows - 1) / a.l1.tile_rows;
    const int nft2 = (a.l2.feat + a.l2.tile_rows - 1) / a.l2.tile_rows;
    // per-expert totals and this chunk's prefix: chunk rows are expert-contiguous, so a warp's
    // loads for one chunk are coalesced; sixteen chunks in flight per thread
    for (int e = tid; e < N; e += blockDim.x) {
      int tot = 0, pre = 0, c = 0;
      for (; c + 16 <= nch; c += 16) {
        int v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __ldcg(a.chunk_counts + (long long)(c + j) * N + e);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          tot += v[j];
          pre += (c + j < b) ? v[j] : 0;
        }
      }
      for (; c < nch; ++c) {
        const int v = __ldcg(a.chunk_counts + (long long)c * N + e);
        tot += v;
        pre += c < b ? v : 0;
      }
      s_off[e] = tot;
      s_base[e] = pre;
      const int ntt = (tot + tile - 1) / tile;
      s_t0[e] = ntt;
      s_u1[e] = ntt * nft1;
      s_u2[e] = ntt * nft2;
    }
    __syncthreads();
    if (b == 0)
      for (int e = tid; e < N; e += blockDim.x) a.counts[e] = s_off[e];
    int tots[4];
    block_scan_excl4(s_off, s_t0, s_u1, s_u2, N, s_warp, tots);
    const int total = tots[0], n_tiles = tots[1], nu1 = tots[2], nu2 = tots[3];
    if (tid == 0) {
      s_off[N] = total;
      s_t0[N] = n_tiles;
      s_u1[N] = nu1;
      s_u2[N] = nu2;
    }
    __syncthreads();
    for (int e = tid; e < N; e += blockDim.x) s_base[e] += s_off[e];
    if (b == 0) {
      for (int e = tid; e <= N; e += blockDim.x) {
        a.offsets[e] = s_off[e];
        a.tile0[e] = s_t0[e];
        a.l1.u0[e] = s_u1[e];
        a.l2.u0[e] = s_u2[e];
      }
      if (tid == 0) {
        *a.l1.num_units = min(nu1, a.l1.max_units);
        *a.l2.num_units = min(nu2, a.l2.max_units);
        if (nu1 > a.l1.max_units || nu2 > a.l2.max_units) atomicOr(a.status, DEV_STATUS_BAD_INDEX);
      }
    }
    __syncthreads();
    // unit lists: units of both lists, spread over the chunk blocks; a unit finds its expert by
    // binary search over the first units (the largest expert whose first unit is <= u)
    {
      const int n1 = min(nu1, a.l1.max_units), n2 = min(nu2, a.l2.max_units);
      for (int i = b * blockDim.x + tid; i < n1 + n2; i += nch * blockDim.x) {
        const bool second = i >= n1;
        const UnitListSpec& L = second ? a.l2 : a.l1;
        const int* u0 = second ? s_u2 : s_u1;
        const int nft = second ? nft2 : nft1;
        const int u = second ? i - n1 : i;
        int lo = 0, hi = N - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (u0[mid] <= u) lo = mid;
          else hi = mid - 1;
        }
        const int ex = lo;
        const int local = u - u0[ex];
        const int tt = local / nft, ft = local - tt * nft;
        const int cnt = s_off[ex + 1] - s_off[ex];
        const int nv = min(L.tile_tokens, cnt - tt * L.tile_tokens);
        int4* dst = reinterpret_cast<int4*>(&L.units[u]);
        dst[0] = make_int4(ex * L.feat + ft * L.tile_rows, s_off[ex] + tt * L.tile_tokens, ft * L.tile_rows,
                           nv | (min(L.tile_rows, L.feat - ft * L.tile_rows) << 16));
        dst[1] = make_int4(s_t0[ex] + tt, 0, 0, 0);
      }
    }
    // stable row assignment of the chunk's (token, slot) pairs: warp w ranks the w-th contiguous
    // part (per-warp expert counts, then per-warp bases on top of the chunk's base)
    const long long a_begin = (long long)t_begin * K, a_end = (long long)t_end * K;
    const long long TK = (long long)a.T * K;
    const long long per = (a_end - a_begin + W - 1) / W;
    const long long s_begin = min(a_end, a_begin + warp * per), s_end = min(a_end, s_begin + per);
    int* my = s_hist + warp * N;
    for (int i = tid; i < W * N; i += blockDim.x) s_hist[i] = 0;
    __syncthreads();
    for (long long a0 = s_begin; a0 < s_end; a0 += 32) {
      const long long ai = a0 + lane;
      const int e = ai < s_end ? a.idx[ai] : -1 - lane;
      const bool e_ok = e >= 0 && e < N;
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      if (e_ok && lane == __ffs(peers) - 1) my[e] += __popc(peers);
      __syncwarp();
    }
    __syncthreads();
    for (int e = tid; e < N; e += blockDim.x) {
      int run = s_base[e];
      for (int w = 0; w < W; ++w) {
        const int v = s_hist[w * N + e];
        s_hist[w * N + e] = run;
        run += v;
      }
    }
    __syncthreads();
    for (long long a0 = s_begin; a0 < s_end; a0 += 32) {
      const long long ai = a0 + lane;
      const bool act = ai < s_end;
      const int e = act ? a.idx[ai] : -1 - lane;
      const float g = act ? a.gate[ai] : 0.f;
      const bool e_ok = e >= 0 && e < N;
      if (act && !e_ok) atomicOr(a.status, DEV_STATUS_BAD_INDEX);
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
          a.row_of[ai] = row;
          a.tok_of_row[row] = (int)(ai / K);
          a.gate_of_row[row] = g;
        } else {
          if (e_ok) atomicOr(a.status, DEV_STATUS_BAD_INDEX);
          a.row_of[ai] = -1;
        }
      }
    }
  }
  if (a.fp4) {
    // x and h quantised with the tensor scales from the grid's maxima: the blocks without a chunk,
    // or every block (after its chunk's work) when all blocks own a chunk
    const int qn = G > nch ? G - nch : G, qb = G > nch ? b - nch : b;
    if (qb >= 0) {
      const float g_x = tensor_scale_from_amax(__uint_as_float(__ldcg(a.amax)));
      const float g_h = tensor_scale_from_amax(__uint_as_float(__ldcg(a.amax + 1)));
      if (qb == 0 && tid == 0) {
        a.act_g[0] = g_x;
        a.act_g[1] = g_h;
      }
      const long long i0 = (long long)qb * blockDim.x + tid, st = (long long)qn * blockDim.x;
      quant_act_blocks<true>(a.x, a.d, nullptr, a.T, a.T, nullptr, nullptr, N, a.tile_tokens4, a.nra4, g_x, a.xq, a.x_sf,
                       a.status, 1, i0, st);
      quant_act_blocks<true>(a.h, l, nullptr, a.T, a.T, nullptr, nullptr, N, a.tile_tokens4, 0, g_h, a.hq_tok, a.h_sf_tok,
                       a.status, 1, i0, st);
    }
  }

  if (!grid_barrier_bounded(a.bar, a.timeout_ns, a.status)) return;

  if (a.fp4) {
    // ------------------------------------------------------------------ phase 3 (NVFP4)
    // the expert offsets and first token tiles, once per block into shared memory: every row's
    // expert search then runs there
    int* s_offm = smem_i;            // [N + 1]
    int* s_t0m = smem_i + (N + 1);   // [N + 1]
    for (int e = tid; e <= N; e += blockDim.x) {
      s_offm[e] = __ldcg(a.offsets + e);
      s_t0m[e] = __ldcg(a.tile0 + e);
    }
    __syncthreads();
    gather_act_q_rows<true, true>(a.hq_tok, a.h_sf_tok, l, a.tok_of_row, (long long)a.T * K, a.T, s_offm, s_t0m, N,
                      a.tile_tokens4, a.nra4, a.hq, a.h_sf, a.status, 1, (long long)b * W + warp, (long long)G * W);
    return;
  }

  // ------------------------------------------------------------------ phase 3
  // h_perm[r] = h[tok_of_row[r]] over the whole grid: a warp copies four rows at a time, all of a
  // lane's 16-byte loads (four per row for a row of up to 1024 bf16) in flight together
  {
    const long long TK = (long long)a.T * K;
    const int vpr = l / 8;  // 16-byte vectors per latent row
    const long long gw = (long long)b * W + warp, nw = (long long)G * W;
    for (long long r0 = gw * 4; r0 < TK; r0 += nw * 4) {
      int tok[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const long long r = r0 + j;
        int t = r < TK ? __ldcg(a.tok_of_row + r) : -1;
        if (r < TK && (t < 0 || t >= a.T)) {
          if (lane == 0) atomicOr(a.status, DEV_STATUS_BAD_INDEX);
          t = -1;
        }
        tok[j] = t;
      }
      for (int c0 = 0; c0 < vpr; c0 += 128) {
        uint4 buf[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int v = 0; v < 4; ++v)
            if (tok[j] >= 0 && c0 + 32 * v + lane < vpr)
              buf[j][v] = __ldcg(reinterpret_cast<const uint4*>(a.h + (long long)tok[j] * l) + c0 + 32 * v + lane);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int v = 0; v < 4; ++v)
            if (tok[j] >= 0 && c0 + 32 * v + lane < vpr)
              reinterpret_cast<uint4*>(a.h_perm + (r0 + j) * l)[c0 + 32 * v + lane] = buf[j][v];
      }
    }
  }
}

}  // namespace lmoe
