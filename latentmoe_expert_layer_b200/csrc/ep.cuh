// Expert parallelism: the device-side parts of a LatentMoE forward spread over G ranks that each own
// N / G consecutive experts ("Nemotron 3 Super" notes, section 3.2: LatentMoE dispatches the latent
// h = W_down x, l wide instead of d, so the all-to-all routing traffic shrinks by d / l).
//
//   source side   ep_plan_kernel         the send plan of a rank's routing: one latent row per
//                                        (token, owner rank) pair, pairs in (destination, token) order;
//                                        per assignment in (destination, token, slot) order its pair
//                                        index within the destination, its expert id local to the
//                                        destination and its gate; per token its pairs' send-order
//                                        indices
//                 ep_gather_send_kernel  the pairs' latent rows into the send buffer
//   owner side    ep_split_meta_kernel   received metadata into local expert ids and source rows
//                 ids_hist_kernel        per-chunk histogram of those expert ids (the single-GPU
//                                        scan / unit-list / stable-row kernels follow)
//                 gather_src_kernel      grouped rows from the received latent rows
//                 ep_pair_reduce_kernel  sum of each pair's gated expert outputs in arrival order
//   source side   ep_combine_kernel      z[t] = the token's returned partial sums in ascending owner
//                                        order
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace lmoe {

constexpr int EP_MAX_WORLD = 8;
constexpr int EP_PLAN_THREADS = 512;

// Exclusive scan over the block of Q values per thread (block of at most 1024 threads); v becomes
// the sum of the lower threads' values, tot the block totals.  s_buf: Q * 33 ints of shared memory.
template <int Q>
__device__ __forceinline__ void block_scan_regs(int (&v)[Q], int (&tot)[Q], int* s_buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl[Q];
#pragma unroll
  for (int q = 0; q < Q; ++q) incl[q] = v[q];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      const int y = __shfl_up_sync(0xffffffffu, incl[q], o);
      if (lane >= o) incl[q] += y;
    }
  if (lane == 31)
#pragma unroll
    for (int q = 0; q < Q; ++q) s_buf[q * 33 + warp] = incl[q];
  __syncthreads();
  if (warp == 0) {
    for (int q = 0; q < Q; ++q) {
      const int w = lane < nw ? s_buf[q * 33 + lane] : 0;
      int ws = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, ws, o);
        if (lane >= o) ws += y;
      }
      if (lane < nw) s_buf[q * 33 + lane] = ws - w;
      if (lane == 31) s_buf[q * 33 + 32] = ws;
    }
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < Q; ++q) {
    const int ex = s_buf[q * 33 + warp] + incl[q] - v[q];
    tot[q] = s_buf[q * 33 + 32];
    v[q] = ex;
  }
  __syncthreads();
}

// One block of EP_PLAN_THREADS threads; each thread owns a contiguous run of tokens.  G <= 8.
//   counts    [G][2]   pairs, assignments per destination
//   send_tok  [T*GP]   token of each pair, send order (entries P.. unused)
//   send_meta [T*K][2] (pair index within the destination, local expert id), send order
//   send_gate [T*K]
//   tok_pairs [T][GP]  send-order pair indices of each token, ascending destination, then -1
// An expert id outside 0..N-1 raises DEV_STATUS_BAD_INDEX and its assignment is not sent.
__global__ void __launch_bounds__(EP_PLAN_THREADS)
    ep_plan_kernel(const int* __restrict__ idx, const float* __restrict__ gate, int T, int K, int n_experts,
                   int per_rank, int G, int GP, int* __restrict__ counts, int* __restrict__ send_tok,
                   int* __restrict__ send_meta, float* __restrict__ send_gate, int* __restrict__ tok_pairs,
                   unsigned* status) {
  __shared__ int s_buf[2 * EP_MAX_WORLD * 33];
  __shared__ int s_off[2][EP_MAX_WORLD];  // first pair / assignment of each destination
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (T + nt - 1) / nt;
  const int t0 = min(T, tid * per), t1 = min(T, t0 + per);
  auto owner = [&](int e) { return (e >= 0 && e < n_experts) ? e / per_rank : -1; };
  // pass 1: per-destination pairs (v[g]) and assignments (v[8 + g]) of this thread's tokens
  int v[2 * EP_MAX_WORLD];
#pragma unroll
  for (int q = 0; q < 2 * EP_MAX_WORLD; ++q) v[q] = 0;
  for (int t = t0; t < t1; ++t) {
    unsigned mask = 0;
    for (int k = 0; k < K; ++k) {
      const int g = owner(idx[(long long)t * K + k]);
      if (g < 0) {
        atomicOr(status, DEV_STATUS_BAD_INDEX);
        continue;
      }
      mask |= 1u << g;
#pragma unroll
      for (int gg = 0; gg < EP_MAX_WORLD; ++gg) v[EP_MAX_WORLD + gg] += (g == gg);
    }
#pragma unroll
    for (int gg = 0; gg < EP_MAX_WORLD; ++gg) v[gg] += (mask >> gg) & 1u;
  }
  int tot[2 * EP_MAX_WORLD];
  block_scan_regs<2 * EP_MAX_WORLD>(v, tot, s_buf);
  if (tid == 0) {
    int p = 0, a = 0;
    for (int g = 0; g < G; ++g) {
      s_off[0][g] = p;
      s_off[1][g] = a;
      counts[2 * g] = tot[g];
      counts[2 * g + 1] = tot[EP_MAX_WORLD + g];
      p += tot[g];
      a += tot[EP_MAX_WORLD + g];
    }
  }
  __syncthreads();
  // pass 2: this thread's tokens in order; v[g] / v[8 + g] now count the pairs / assignments of
  // destination g that lower threads send
  for (int t = t0; t < t1; ++t) {
    unsigned mask = 0;
    for (int k = 0; k < K; ++k) {
      const int g = owner(idx[(long long)t * K + k]);
      if (g >= 0) mask |= 1u << g;
    }
    int j = 0;
    for (int g = 0; g < G; ++g) {
      if (!((mask >> g) & 1u)) continue;
      int pg = 0, ag = 0;
#pragma unroll
      for (int gg = 0; gg < EP_MAX_WORLD; ++gg)
        if (gg == g) {
          pg = v[gg]++;
          ag = v[EP_MAX_WORLD + gg];
        }
      const int P = s_off[0][g] + pg;
      send_tok[P] = t;
      tok_pairs[(long long)t * GP + j++] = P;
      int na = 0;
      for (int k = 0; k < K; ++k) {
        const int e = idx[(long long)t * K + k];
        if (owner(e) != g) continue;
        const long long A = s_off[1][g] + ag + na++;
        send_meta[2 * A] = pg;
        send_meta[2 * A + 1] = e - g * per_rank;
        send_gate[A] = gate[(long long)t * K + k];
      }
#pragma unroll
      for (int gg = 0; gg < EP_MAX_WORLD; ++gg)
        if (gg == g) v[EP_MAX_WORLD + gg] += na;
    }
    for (; j < GP; ++j) tok_pairs[(long long)t * GP + j] = -1;
  }
}

// send_rows[P] = h[send_tok[P]] for P < the plan's pair total (counts[0..G) pairs); one warp per row.
__global__ void __launch_bounds__(256)
    ep_gather_send_kernel(const __nv_bfloat16* __restrict__ h, const int* __restrict__ send_tok,
                          const int* __restrict__ counts, int G, int T, int l, __nv_bfloat16* __restrict__ send_rows,
                          unsigned* status) {
  int P = 0;
  for (int g = 0; g < G; ++g) P += counts[2 * g];
  const int lane = threadIdx.x & 31;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int vpr = l / 8;
  for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < P; r += nwarps) {
    const int t = send_tok[r];
    if (t < 0 || t >= T) {
      if (lane == 0) atomicOr(status, DEV_STATUS_BAD_INDEX);
      continue;
    }
    for (int i = lane; i < vpr; i += 32)
      reinterpret_cast<uint4*>(send_rows + r * l)[i] = reinterpret_cast<const uint4*>(h + (long long)t * l)[i];
  }
}

// Received metadata [A][2] = (source row, local expert) into ids[A] and src[A].
__global__ void ep_split_meta_kernel(const int* __restrict__ meta, long long A, int* __restrict__ ids,
                                     int* __restrict__ src) {
  for (long long a = (long long)blockIdx.x * blockDim.x + threadIdx.x; a < A; a += (long long)gridDim.x * blockDim.x) {
    src[a] = meta[2 * a];
    ids[a] = meta[2 * a + 1];
  }
}

// Per-chunk expert histogram of ids [n] (chunk c = ids [c * chunk, (c + 1) * chunk)); expert-major
// [N][n_chunks] like topk_hist_kernel's, for scan_units_kernel.  Ids outside 0..N-1 are counted by
// no expert (the stable-row kernel flags them).
__global__ void ids_hist_kernel(const int* __restrict__ ids, long long n, int n_experts, int chunk,
                                int* __restrict__ chunk_counts) {
  extern __shared__ int s_cnt[];
  for (int e = threadIdx.x; e < n_experts; e += blockDim.x) s_cnt[e] = 0;
  __syncthreads();
  const long long a0 = (long long)blockIdx.x * chunk, a1 = min(n, a0 + chunk);
  for (long long a = a0 + threadIdx.x; a < a1; a += blockDim.x) {
    const int e = ids[a];
    if (e >= 0 && e < n_experts) atomicAdd(&s_cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n_experts; e += blockDim.x)
    chunk_counts[(long long)e * gridDim.x + blockIdx.x] = s_cnt[e];
}

// h_perm[r] = rows[src[tok_of_row[r]]] for the n grouped rows; one warp per row.
__global__ void __launch_bounds__(256)
    gather_src_kernel(const __nv_bfloat16* __restrict__ rows, int n_src_rows, const int* __restrict__ src,
                      const int* __restrict__ tok_of_row, long long n, long long n_assign, int l,
                      __nv_bfloat16* __restrict__ h_perm, unsigned* status) {
  const int lane = threadIdx.x & 31;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int vpr = l / 8;
  for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < n; r += nwarps) {
    const int a = tok_of_row[r];
    const int s = (a >= 0 && a < n_assign) ? src[a] : -1;
    if (s < 0 || s >= n_src_rows) {
      if (lane == 0) atomicOr(status, DEV_STATUS_BAD_INDEX);
      continue;
    }
    for (int i = lane; i < vpr; i += 32)
      reinterpret_cast<uint4*>(h_perm + r * l)[i] = reinterpret_cast<const uint4*>(rows + (long long)s * l)[i];
  }
}

// partial[r] = sum, in arrival order, of o[row_of[a]] over the assignments a with src[a] == r (src is
// nondecreasing, so they are contiguous); fp32, eight columns per thread.  Rows without assignments
// get zeros.
__global__ void __launch_bounds__(256)
    ep_pair_reduce_kernel(const __nv_bfloat16* __restrict__ o, const int* __restrict__ row_of,
                          const int* __restrict__ src, long long n_assign, long long n_grouped, int R, int l,
                          float* __restrict__ partial, unsigned* status) {
  const int vpr = l / 8;
  const long long total = (long long)R * vpr;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / vpr), v = (int)(i % vpr);
    long long lo = 0, hi = n_assign;  // first assignment with src >= r
    while (lo < hi) {
      const long long mid = (lo + hi) >> 1;
      if (src[mid] < r) lo = mid + 1;
      else hi = mid;
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (long long a = lo; a < n_assign && src[a] == r; ++a) {
      const int row = row_of[a];
      if (row < 0 || row >= n_grouped) {
        atomicOr(status, DEV_STATUS_BAD_INDEX);
        continue;
      }
      const uint4 q = *reinterpret_cast<const uint4*>(o + (long long)row * l + v * 8);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(p[j]);
        acc[2 * j] += f.x;
        acc[2 * j + 1] += f.y;
      }
    }
    float4* dst = reinterpret_cast<float4*>(partial + (long long)r * l + v * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

// z[t] = bf16(sum over j of back[tok_pairs[t][j]]), pairs in ascending owner order, -1 ends the list;
// fp32 accumulation, eight columns per thread, written to zu[t, 0:l].
__global__ void __launch_bounds__(256)
    ep_combine_kernel(const float* __restrict__ back, int n_back, const int* __restrict__ tok_pairs, int T, int GP,
                      int l, __nv_bfloat16* __restrict__ zu, long long ld_zu, unsigned* status) {
  const int vpr = l / 8;
  const long long total = (long long)T * vpr;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long t = i / vpr;
    const int v = (int)(i % vpr);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < GP; ++j) {
      const int p = tok_pairs[t * GP + j];
      if (p < 0) break;
      if (p >= n_back) {
        atomicOr(status, DEV_STATUS_BAD_INDEX);
        continue;
      }
      const float4* src = reinterpret_cast<const float4*>(back + (long long)p * l + v * 8);
      const float4 a = src[0], b = src[1];
      acc[0] += a.x;
      acc[1] += a.y;
      acc[2] += a.z;
      acc[3] += a.w;
      acc[4] += b.x;
      acc[5] += b.y;
      acc[6] += b.z;
      acc[7] += b.w;
    }
    uint4 out;
    __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
    for (int j = 0; j < 4; ++j) po[j] = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
    *reinterpret_cast<uint4*>(zu + t * ld_zu + v * 8) = out;
  }
}

}  // namespace lmoe
