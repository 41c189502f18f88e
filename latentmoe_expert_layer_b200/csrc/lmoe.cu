// Host side of the LatentMoE layer library: argument checking, workspace, weight preparation,
// tensor maps and the launch sequence of one forward pass.  Everything on the path runs in the
// kernels of this directory; the host only validates, enqueues and reports.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/lmoe.h"
#include "ep.cuh"
#include "gemm_tc.cuh"
#include "route_fused.cuh"
#include "routing.cuh"

using namespace lmoe;

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool load_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// 2-D bf16 tensor map over rows x cols (row pitch ld elements), 64-element x box_rows tiles,
// 128-byte swizzle (the layout the MMA descriptors expect).
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// GEMM shapes: small token tiles with a deep ring (weight streaming at decode sizes) and large token
// tiles (tensor-core bound at prefill sizes), each in bf16 and in NVFP4.  The bf16 large-tile variant
// runs as CTA pairs (cta_group::2 MMAs over 256 weight rows x 256 tokens; each CTA loads 128 weight
// rows and 128 tokens per stage).  V_LARGE1 is the same token tile on one CTA with 128 weight rows:
// the prefill expert-up GEMM uses it, because its 2688 features would leave half of every 11th pair
// tile empty (measured: the pair variant was 7 % slower there, the down GEMM and the dense GEMMs
// faster).
enum Variant { V_SMALL = 0, V_LARGE = 1, V_SMALL4 = 2, V_LARGE4 = 3, V_LARGE1 = 4 };
constexpr int V_BN[5] = {64, 256, 64, 192, 256};
constexpr int V_STAGES[5] = {8, 6, 6, 3, 4};
constexpr int V_BOXN[5] = {16, 128, 16, 192, 256};  // one token box per stage (per CTA) at prefill sizes
constexpr bool V_FP4[5] = {false, false, true, true, false};
constexpr int V_ACC_SPLIT[5] = {4, 1, 2, 1, 1};  // decode-sized tiles rotate over independent accumulators
// K stages of one token tile's activation scales that fit resident in TMEM (0: per-stage copies)
constexpr int V_RES[5] = {0, 0, 12, 0, 0};
constexpr bool V_PAIR[5] = {false, true, false, false, false};
// epilogue warps: eight for the NVFP4 prefill variant, whose fc1 epilogue (squared ReLU and the NVFP4
// quantisation of u) costs more than the MMAs of a K = 1024 unit
constexpr int V_EPIW[5] = {4, 4, 4, 8, 4};
constexpr int V_TILE_M[5] = {128, 256, 128, 128, 128};  // weight rows per unit

template <int V>
struct VT {
  static constexpr int BN = V_BN[V], ST = V_STAGES[V], BOX = V_BOXN[V], AS = V_ACC_SPLIT[V], RS = V_RES[V];
  static constexpr bool F4 = V_FP4[V], PR = V_PAIR[V];
  static constexpr int EW = V_EPIW[V], THREADS = 64 + 32 * V_EPIW[V];
  static void* fn() { return reinterpret_cast<void*>(gemm_tc_kernel<BN, ST, BOX, F4, AS, RS, PR, EW>); }
  static int smem() { return GemmSmem<BN, ST, F4, AS, RS, PR, EW>::ALLOC; }
};

// 2-D byte tensor map (packed NVFP4 codes): rows x cols_bytes, 128-byte x box_rows tiles, 128-byte swizzle.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols_bytes, uint64_t ld_bytes,
                 uint32_t box_rows) {
  cuuint64_t dims[2] = {cols_bytes, rows};
  cuuint64_t strides[1] = {ld_bytes};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded wait

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

struct lmoe_ctx {
  lmoe_config cfg{};
  int device = 0;
  int num_sms = 148;
  int pair_workers = 74;  // CTA pairs of the pair variant that can be resident at once
  bool loaded = false;
  bool router_f32 = false;
  bool fused_router = false;
  bool standard = false;  // latent == 0: a standard MoE, experts d -> m -> d, no W_down / W_up
  int le = 0;             // width the routed experts work in: latent, or d for a standard MoE
  int ep_world = 0;       // expert parallelism: G ranks (>= 2), this one ep_rank, owning n_local experts
  int ep_rank = 0;
  int n_local = 0;        // experts whose weights this handle holds (N, or N / G)
  long long tk_exp = 0;   // capacity in assignments of the expert-side buffers
  unsigned long long timeout_ns = kDefaultTimeoutNs;

  // weights (library-owned)
  __nv_bfloat16* w_rd = nullptr;   // [N + l, d]: router rows then W_down rows (bf16 router)
  float* w_r32 = nullptr;          // [N, d] fp32 router
  __nv_bfloat16* w_down = nullptr; // [l, d] when not stacked with the router
  float* b_router = nullptr;       // [N]
  __nv_bfloat16* w_cat = nullptr;  // [d, l + m_s]: W_up columns then W_s2 columns
  __nv_bfloat16* ws1 = nullptr;    // [m_s, d]
  __nv_bfloat16* w1 = nullptr;     // [N * m, l]
  __nv_bfloat16* w2 = nullptr;     // [N * l, m]
  CUtensorMap map_rd{}, map_r{}, map_down{}, map_cat{}, map_ws1{}, map_w1{}, map_w2{};
  CUtensorMap map_wup{}, map_ws2{};  // the W_up and W_s2 column blocks of w_cat

  // workspace
  float* logits = nullptr;
  int* idx = nullptr;
  float* gate = nullptr;
  int* chunk_counts = nullptr;
  int* chunk_base = nullptr;
  int* counts = nullptr;
  int* offsets = nullptr;
  int* row_of = nullptr;
  int* tok_of_row = nullptr;
  float* gate_of_row = nullptr;
  __nv_bfloat16* h = nullptr;
  __nv_bfloat16* h_perm = nullptr;
  __nv_bfloat16* u = nullptr;
  __nv_bfloat16* o = nullptr;
  __nv_bfloat16* zu = nullptr;
  GemmUnit* units1 = nullptr;
  GemmUnit* units2 = nullptr;
  int* num_units = nullptr;  // [2]
  unsigned* status = nullptr;
  unsigned* route_bar = nullptr;  // [2] grid barrier of the fused decode routing kernel (zero at rest)
  int* ep_ids = nullptr;          // [tk_exp] expert parallelism: received assignments' local experts
  int* ep_src = nullptr;          // [tk_exp] and their rows in the received latent rows
  int* ep_send_tok = nullptr;     // [max_tokens * min(K, G)] token of each sent pair
  int* work_counters = nullptr;  // [kCounters] per-launch unit counters and (last two) activation amax
                                 // bits, all zeroed at the start of a forward
  static constexpr int kCounters = 10;
  static constexpr int kAmaxX = 8, kAmaxH = 9;
  int max_units1 = 0, max_units2 = 0;
  CUtensorMap map_hperm[2]{}, map_u[2]{}, map_zu[2]{};
  CUtensorMap map_hperm1{};  // h_perm with the single-CTA large token tile (expert up, V_LARGE1)
  CUtensorMap map_z[2]{}, map_us[2]{};  // the z and u_s column blocks of zu
  float* y_s = nullptr;                 // [min(T_max, 512), d] fp32: W_s2 u_s at decode sizes

  // x tensor maps, cached by (pointer, T)
  const void* x_cached = nullptr;
  int x_cached_T = -1;
  CUtensorMap map_x[2]{};

  // staging for lmoe_forward_host
  __nv_bfloat16* x_dev = nullptr;
  __nv_bfloat16* y_dev = nullptr;
  int* idx_dev = nullptr;
  float* gate_dev = nullptr;
  // chunked host forward: copy streams and their events (created on first use)
  cudaStream_t host_in = nullptr, host_out = nullptr;
  std::vector<cudaEvent_t> host_ev;

  int last_T = 0;

  // NVFP4 (precision == LMOE_PREC_NVFP4): weights, scales, activation buffers
  bool nvfp4 = false;
  uint8_t *w1q = nullptr, *w2q = nullptr, *ws1q = nullptr, *ws2q = nullptr;          // codes
  uint8_t *w1_sf = nullptr, *w2_sf = nullptr, *ws1_sf = nullptr, *ws2_sf = nullptr;  // scale atoms
  float* wg = nullptr;            // tensor scales: [0, N) W1, [N, 2N) W2, 2N W_s1, 2N + 1 W_s2
  unsigned* w_amax = nullptr;     // [2N + 2] amax bits used while quantising
  uint8_t *xq = nullptr, *x_sf = nullptr, *hq = nullptr, *h_sf = nullptr;  // x [T, d]; h grouped [TK, l]
  uint8_t *hq_tok = nullptr, *h_sf_tok = nullptr;  // h per token [T, l/2] codes, [T, l/16] plain scales
  uint8_t *uq = nullptr, *u_sf = nullptr, *usq = nullptr, *us_sf = nullptr; // u [TK, m]; u_s [T, m_s]
  float* act_g = nullptr;         // [0] g_x, [1] g_h, [2] 1.0
  int* tile0 = nullptr;           // [N + 1] first token tile of each expert
  int* unit_u0 = nullptr;         // [2][N + 1] first unit of each expert in the two unit lists
  // router K-slice partials, fp32 [slices][T][N + l] at decode sizes (T <= kSplitRows), [slices][T][N]
  // above
  float* router_part = nullptr;
  static constexpr int kSplitRows = 512, kMaxSplits = 8;
  CUtensorMap map_w1q{}, map_w2q{}, map_ws1q{}, map_ws2q{};
  CUtensorMap map_xq[4]{}, map_hq[4]{}, map_uq[4]{}, map_usq[4]{};  // indexed by variant (FP4 ones)

  // Bytes of tile-local activation scales for K-extent K, large enough for either FP4 variant:
  // tiles x stages x 4 K atoms x row atoms x 512.  Dense tensors tile T_max tokens; grouped ones have
  // at most N + T_max*K / tile_tokens tiles.
  size_t sf_bytes_tiles(long long tiles_small, long long tiles_large, int K) const {
    const long long st = (K + NVFP4_STAGE_K - 1) / NVFP4_STAGE_K;
    const long long a = tiles_small * st * 4 * ((V_BN[V_SMALL4] + 127) / 128) * 512;
    const long long b = tiles_large * st * 4 * ((V_BN[V_LARGE4] + 127) / 128) * 512 * SF_WREP;  // replicated
    return (size_t)(a > b ? a : b);
  }
  size_t sf_bytes_dense(int K) const {
    const long long T = cfg.max_tokens;
    return sf_bytes_tiles((T + V_BN[V_SMALL4] - 1) / V_BN[V_SMALL4], (T + V_BN[V_LARGE4] - 1) / V_BN[V_LARGE4], K);
  }
  size_t sf_bytes_grouped(int K) const {
    const long long tk = (long long)cfg.max_tokens * cfg.top_k, n = cfg.n_experts;
    return sf_bytes_tiles(n + (tk + V_BN[V_SMALL4] - 1) / V_BN[V_SMALL4], n + (tk + V_BN[V_LARGE4] - 1) / V_BN[V_LARGE4],
                          K);
  }

  // stage profiler
  static constexpr int kProfMax = 1024;
  bool prof_on = false;
  int prof_n = 0;
  int launches = 0;
  std::vector<cudaEvent_t> prof_ev;  // kProfMax x (LMOE_NUM_STAGES + 1)
};

namespace {

// Makes `dev` current for the call, restoring the caller's device afterwards.  cudaSetDevice runs even
// when the device is already current: it also binds the device's primary context to the calling
// host thread, which the driver-API tensor-map encoder needs (a thread that has made no runtime call
// yet has no current context).
struct DeviceGuard {
  int prev = -1;
  int dev;
  explicit DeviceGuard(int d) : dev(d) {
    cudaGetDevice(&prev);
    cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    if (prev >= 0 && prev != dev) cudaSetDevice(prev);
  }
};

template <typename T>
bool dalloc(T** p, size_t elems) {
  *p = nullptr;
  if (elems == 0) elems = 1;
  return cudaMalloc(reinterpret_cast<void**>(p), elems * sizeof(T)) == cudaSuccess;
}

void free_all(lmoe_ctx* c) {
  void* ptrs[] = {c->w_rd,   c->w_r32,  c->w_down, c->b_router,  c->w_cat,      c->ws1,        c->w1,
                  c->w2,     c->logits, c->idx,    c->gate,      c->chunk_counts, c->chunk_base, c->counts,
                  c->offsets, c->row_of, c->tok_of_row, c->gate_of_row, c->h, c->h_perm, c->u,
                  c->o,      c->zu,     c->units1, c->units2,    c->num_units,  c->status,     c->x_dev,
                  c->y_dev,  c->idx_dev, c->gate_dev, c->y_s, c->work_counters,
                  c->w1q,    c->w2q,    c->ws1q,   c->ws2q,      c->w1_sf,      c->w2_sf,      c->ws1_sf,
                  c->ws2_sf, c->wg,     c->w_amax, c->xq,        c->x_sf,       c->hq,         c->h_sf,
                  c->hq_tok, c->h_sf_tok,
                  c->uq,     c->u_sf,   c->usq,    c->us_sf,     c->act_g,      c->tile0,      c->unit_u0,
                  c->router_part, c->route_bar, c->ep_ids, c->ep_src, c->ep_send_tok};
  for (void* p : ptrs)
    if (p) cudaFree(p);
}

// Tokens are routed in chunks (one top-K block per chunk); the [N][chunks] histogram must fit the
// scan kernel's shared memory, so N * chunks <= 32768, and there are at most 128 chunks.
int n_chunks_for(int T, int N, int* chunk_tokens) {
  int cap = 32768 / N;
  if (cap > 128) cap = 128;
  if (cap < 1) cap = 1;
  int c = (T + 7) / 8;
  if (c > cap) c = cap;
  if (c < 1) c = 1;
  const int ct = (T + c - 1) / c;
  *chunk_tokens = ct;
  return (T + ct - 1) / ct;
}

// blocks per token chunk of the top-K kernel: chunks of more than 32 tokens are split so that a
// warp selects for about one token (the chunk count is capped by the scan's shared memory)
int topk_parts(int chunk_tokens) {
  int p = chunk_tokens / 32;
  return p < 1 ? 1 : (p > 16 ? 16 : p);
}

constexpr int kScanSmemMax = 200 * 1024;

lmoe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA; }

template <int V>
cudaError_t launch_gemm_v(const CUtensorMap& w0, const CUtensorMap& a0, const CUtensorMap& w1, const CUtensorMap& a1,
                          const GemmArgs& a, int grid, cudaStream_t s) {
  return launch_pdl(
      gemm_tc_kernel<VT<V>::BN, VT<V>::ST, VT<V>::BOX, VT<V>::F4, VT<V>::AS, VT<V>::RS, VT<V>::PR, VT<V>::EW>, grid,
      VT<V>::THREADS, VT<V>::smem(), s, VT<V>::PR ? 2 : 1, w0, a0, w1, a1, a);
}

// A bf16 problem with its epilogue; K in elements (multiple of 64).
GemmProblem problem(int K, int epi, void* out, long long ldo, int col0 = 0) {
  GemmProblem p;
  memset(&p, 0, sizeof(p));
  p.num_k_blocks = K / BLOCK_K;
  p.epi = epi;
  p.out = out;
  p.ldo = ldo;
  p.out_col0 = col0;
  return p;
}

// An NVFP4 problem: K in elements; weight scale atoms / tensor scales; activation scales.
GemmProblem problem4(int K, int epi, void* out, long long ldo, const uint8_t* w_sf, const float* w_g,
                     int w_rows_per_g, const uint8_t* act_sf, const float* act_g) {
  GemmProblem p;
  memset(&p, 0, sizeof(p));
  p.num_k_blocks = (K + NVFP4_STAGE_K - 1) / NVFP4_STAGE_K;
  p.epi = epi;
  p.out = out;
  p.ldo = ldo;
  p.w_sf = w_sf;
  p.w_atoms_k = sf_atoms_k(K);
  p.w_gscale = w_g;
  p.w_rows_per_g = w_rows_per_g;
  p.act_sf = act_sf;
  p.act_sf_stages = p.num_k_blocks;
  p.act_gscale = act_g;
  return p;
}

// Make `p` a dense problem over feat x tokens with the token tile of variant v.
int set_dense(GemmProblem& p, int v, int feat, int tokens) {
  p.dense_ftiles = (feat + V_TILE_M[v] - 1) / V_TILE_M[v];
  p.dense_ttiles = (tokens + V_BN[v] - 1) / V_BN[v];
  p.dense_feat = feat;
  p.dense_tokens = tokens;
  p.weights_streamed = p.dense_ttiles == 1;
  return p.dense_ftiles * p.dense_ttiles * (p.k_splits > 1 ? p.k_splits : 1);
}

struct GemmLaunch {
  lmoe_ctx* c;
  int v;
  GemmArgs a;
  const CUtensorMap *w0 = nullptr, *a0 = nullptr, *w1 = nullptr, *a1 = nullptr;

  GemmLaunch(lmoe_ctx* ctx, int variant, int counter) : c(ctx), v(variant) {
    memset(&a, 0, sizeof(a));
    a.status = ctx->status;
    a.timeout_ns = ctx->timeout_ns;
    a.work_counter = ctx->work_counters + counter;
    a.chunk = 1;
  }
  // main problem, dense
  void main_dense(const CUtensorMap& mw, const CUtensorMap& ma, GemmProblem p, int feat, int tokens) {
    a.main_dense_units = set_dense(p, v, feat, tokens);
    a.prob[0] = p;
    w0 = &mw;
    a0 = &ma;
  }
  // main problem, grouped experts (unit list on the device)
  // feat: output features of every expert (units per token tile = ceil(feat / 128));
  // max_tiles: upper bound on the token tiles of the launch
  void main_grouped(const CUtensorMap& mw, const CUtensorMap& ma, GemmProblem p, const GemmUnit* units,
                    const int* num_units, int feat, long long max_tiles) {
    const bool small = v == V_SMALL || v == V_SMALL4;
    p.weights_streamed = small;  // decode-sized groups: mostly one token tile per expert
    a.dynamic = small;           // measured: dynamic claiming helps decode-sized groups only
    if (V_FP4[v] && p.num_k_blocks <= V_RES[v]) {
      // A token tile's activation scales stay in TMEM while a claim's units use that tile.  A claim
      // is a divisor of the tile's feature-tile count (claims never straddle two tiles), as large
      // as leaves every CTA about 6 claims to balance the load with.
      p.sfb_resident = 1;
      const int nft = (feat + BLOCK_M - 1) / BLOCK_M;
      const long long cap = max_tiles * nft / (6LL * c->num_sms);
      int ch = 1;
      for (int cand = nft; cand >= 1; --cand)
        if (nft % cand == 0 && cand <= cap) {
          ch = cand;
          break;
        }
      a.chunk = ch;
    }
    a.prob[0] = p;
    a.units = units;
    a.num_units = num_units;
    w0 = &mw;
    a0 = &ma;
  }
  // dense pre problem, processed before the main problem's units
  void pre_dense(const CUtensorMap& mw, const CUtensorMap& ma, GemmProblem p, int feat, int tokens) {
    a.n_pre_units = set_dense(p, v, feat, tokens);
    a.prob[1] = p;
    w1 = &mw;
    a1 = &ma;
  }
  cudaError_t run(cudaStream_t s) {
    if (!w1) {
      w1 = w0;
      a1 = a0;
    }
    // one worker per SM, or per pair of SMs for the pair variant (grid = 2 x workers)
    const int per = V_PAIR[v] ? 2 : 1;
    int grid = V_PAIR[v] ? c->pair_workers : c->num_sms;
    if (a.units == nullptr) {
      const int total = a.n_pre_units + a.main_dense_units;
      if (total < grid) grid = total;
    }
    if (grid < 1) grid = 1;
    grid *= per;
    switch (v) {
      case V_SMALL: return launch_gemm_v<V_SMALL>(*w0, *a0, *w1, *a1, a, grid, s);
      case V_LARGE: return launch_gemm_v<V_LARGE>(*w0, *a0, *w1, *a1, a, grid, s);
      case V_SMALL4: return launch_gemm_v<V_SMALL4>(*w0, *a0, *w1, *a1, a, grid, s);
      case V_LARGE1: return launch_gemm_v<V_LARGE1>(*w0, *a0, *w1, *a1, a, grid, s);
      default: return launch_gemm_v<V_LARGE4>(*w0, *a0, *w1, *a1, a, grid, s);
    }
  }
};

// warps per token chunk of the stable row assignment (each ranks a contiguous part of the chunk)
constexpr int kAssignWarps = 8;

// Router logits are sums of at least kRouterPartials independent fp32 partial accumulators.  The
// tensor core's fp32 accumulation error grows linearly with the length of one accumulation chain
// (measured on B200 over K = 4096 with N(0, 1) logits: max error 3.0e-5, 6.7e-6, 2.9e-6 and 1.9e-6
// with 1, 4, 8 and 16 partials), while a routing decision is trusted only down to logit gaps of
// 1e-5.  Partials come from K slices (fp32 slice sums by split_reduce_kernel) times the GEMM
// variant's interleaved accumulators (V_ACC_SPLIT).
constexpr int kRouterPartials = 8;

// K slices of the router GEMM: enough for kRouterPartials partials, and at decode sizes as many as
// fill the GPU (one SM streams only ~1/148 of HBM bandwidth); never an empty slice.
int router_splits(const lmoe_ctx* c, int T, int v, int units_per_slice) {
  const int nkb = c->cfg.d / BLOCK_K;
  const int need = (kRouterPartials + V_ACC_SPLIT[v] - 1) / V_ACC_SPLIT[v];
  int ks = v == V_SMALL ? c->num_sms / units_per_slice : need;
  if (ks < need) ks = need;
  if (ks > lmoe_ctx::kMaxSplits) ks = lmoe_ctx::kMaxSplits;
  if (ks > nkb) ks = nkb;
  const int per = (nkb + ks - 1) / ks;
  return (nkb + per - 1) / per;
}

cudaError_t launch_split_reduce(lmoe_ctx* c, int ks, long long stride, int T, int n_logits, int n_h, cudaStream_t s) {
  const long long work = (long long)T * (n_logits + n_h) / 4;
  long long blocks = (work + 255) / 256;
  if (blocks > 4LL * c->num_sms) blocks = 4LL * c->num_sms;
  split_reduce_kernel<<<(int)blocks, 256, 0, s>>>(c->router_part, ks, stride, T, n_logits, n_h, c->logits, c->h);
  return cudaGetLastError();
}

// Stage 1 of a forward: fp32 router logits and the bf16 latent h = W_down x (none for a standard
// MoE).  `launches` counts the kernels enqueued.
//   fp32 router          CUDA-core fp32 FMAs, then W_down as its own GEMM
//   bf16, decode sizes   one K-sliced GEMM over the stacked [W_r; W_down] rows (or W_r alone), and
//                        the slice sum writes the logits and h
//   bf16, larger T       one launch: W_down (EPI_BF16 into h) as its dense pre problem, the router
//                        rows K-sliced into fp32 partials as its main problem; then the slice sum
//   defer_sum: at decode sizes with the stacked rows, leave the slice sum to the fused routing kernel
//   (only the GEMM is enqueued; *ks_out receives its slice count)
cudaError_t router_stage(lmoe_ctx* c, const void* x, int T, cudaStream_t s, int& launches, bool defer_sum = false,
                         int* ks_out = nullptr) {
  const lmoe_config& g = c->cfg;
  const int N = g.n_experts, l = g.latent, d = g.d;
  const int vd = T <= 512 ? V_SMALL : V_LARGE;
  const int nft_r = (N + BLOCK_M - 1) / BLOCK_M;
  const int ntt = (T + V_BN[vd] - 1) / V_BN[vd];
  cudaError_t e;
  if (c->router_f32) {
    router_f32_kernel<<<T, 256, d * sizeof(float), s>>>(reinterpret_cast<const __nv_bfloat16*>(x), c->w_r32, d, N,
                                                        c->logits);
    e = cudaGetLastError();
    ++launches;
    if (e != cudaSuccess || c->standard) return e;
    GemmLaunch gl(c, vd, 2);
    gl.main_dense(c->map_down, c->map_x[vd], problem(d, EPI_BF16, c->h, l), l, T);
    ++launches;
    return gl.run(s);
  }
  if (vd == V_SMALL && (c->fused_router || c->standard)) {
    // every output row of the GEMM is K-sliced: stacked router + W_down rows, or the router alone
    const int rows = c->fused_router ? N + l : N;
    const int ks = router_splits(c, T, vd, ((rows + BLOCK_M - 1) / BLOCK_M) * ntt);
    GemmLaunch gl(c, vd, 0);
    GemmProblem p = problem(d, EPI_F32, c->router_part, rows);
    p.k_splits = ks;
    p.split_stride = (long long)T * rows;
    gl.main_dense(c->fused_router ? c->map_rd : c->map_r, c->map_x[vd], p, rows, T);
    if ((e = gl.run(s)) != cudaSuccess) return e;
    if (ks_out) *ks_out = ks;
    if (defer_sum && c->fused_router) {
      launches += 1;
      return cudaSuccess;
    }
    launches += 2;
    return launch_split_reduce(c, ks, p.split_stride, T, N, rows - N, s);
  }
  // router rows K-sliced as the main problem, W_down (full K, bf16 out) as the pre problem
  const int ks = router_splits(c, T, vd, nft_r * ntt);
  GemmLaunch gl(c, vd, 0);
  if (!c->standard) gl.pre_dense(c->map_down, c->map_x[vd], problem(d, EPI_BF16, c->h, l), l, T);
  GemmProblem p = problem(d, EPI_F32, c->router_part, N);
  p.k_splits = ks;
  p.split_stride = (long long)T * N;
  gl.main_dense(c->map_r, c->map_x[vd], p, N, T);
  gl.a.dynamic = 1;  // full-K W_down units and 1/ks-K router units: claims balance the mix
  if ((e = gl.run(s)) != cudaSuccess) return e;
  launches += 2;
  return launch_split_reduce(c, ks, p.split_stride, T, N, 0, s);
}

// Tensor maps of the activations x [T, d] for both bf16 variants, cached by (pointer, T).
bool set_x_maps(lmoe_ctx* c, const void* x, int T) {
  if (x == c->x_cached && T == c->x_cached_T) return true;
  for (int v = 0; v < 2; ++v)
    if (!make_map(&c->map_x[v], x, T, c->cfg.d, c->cfg.d, V_BOXN[v])) return false;
  c->x_cached = x;
  c->x_cached_T = T;
  return true;
}

// The two grouped-GEMM unit lists from the scan's first units: one unit per thread.
cudaError_t launch_build_units(const lmoe_ctx* c, cudaStream_t s, const UnitListSpec& l1, const UnitListSpec& l2,
                               int n_experts) {
  const long long cap = (long long)c->max_units1 + c->max_units2;
  long long blocks = (cap + 255) / 256;
  if (blocks > 4LL * c->num_sms) blocks = 4LL * c->num_sms;
  build_units_kernel<<<(int)blocks, 256, 0, s>>>(c->counts, c->offsets, c->tile0, n_experts, l1, l2);
  return cudaGetLastError();
}

// The decode routing chain as one cooperative launch (route_fused.cuh): slice sum of the router
// GEMM (ks slices), top-K, expert scan, unit lists, stable rows and the gather into h_perm; it also
// zeroes the unit counters of the expert launches that follow.
constexpr int kRouteFusedThreads = 256;

template <int P>
cudaError_t launch_route_fused_p(const RouteFusedArgs& a, int grid, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kRouteFusedThreads);
  cfg.dynamicSmemBytes = route_fused_smem(a.N, kRouteFusedThreads / 32);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, route_fused_kernel<P>, a);
}

// fp4_x: NVFP4 experts (the layer input x, quantised here with h); nullptr for bf16 experts.
cudaError_t launch_route_fused(lmoe_ctx* c, int T, int ks, int nch, int ct, int* idx, float* gate,
                               const UnitListSpec& l1, const UnitListSpec& l2, cudaStream_t s,
                               const void* fp4_x = nullptr) {
  const lmoe_config& g = c->cfg;
  RouteFusedArgs a;
  memset(&a, 0, sizeof(a));
  a.part = c->router_part;
  a.ks = ks;
  a.slice_stride = (long long)T * (g.n_experts + g.latent);
  a.bias = c->b_router;
  a.T = T;
  a.N = g.n_experts;
  a.K = g.top_k;
  a.l = g.latent;
  a.chunk_tokens = ct;
  a.n_chunks = nch;
  a.logits = c->logits;
  a.h = c->h;
  a.idx = idx;
  a.gate = gate;
  a.chunk_counts = c->chunk_counts;
  a.counts = c->counts;
  a.offsets = c->offsets;
  a.tile0 = c->tile0;
  a.l1 = l1;
  a.l2 = l2;
  a.row_of = c->row_of;
  a.tok_of_row = c->tok_of_row;
  a.gate_of_row = c->gate_of_row;
  a.h_perm = c->h_perm;
  a.zero_words = c->work_counters;
  a.n_zero = lmoe_ctx::kAmaxX;  // the unit counters (the activation maxima are zeroed before the launch)
  if (fp4_x) {
    a.fp4 = 1;
    a.x = reinterpret_cast<const __nv_bfloat16*>(fp4_x);
    a.d = g.d;
    a.amax = reinterpret_cast<unsigned*>(c->work_counters + lmoe_ctx::kAmaxX);
    a.act_g = c->act_g;
    a.xq = c->xq;
    a.x_sf = c->x_sf;
    a.hq_tok = c->hq_tok;
    a.h_sf_tok = c->h_sf_tok;
    a.hq = c->hq;
    a.h_sf = c->h_sf;
    a.tile_tokens4 = l1.tile_tokens;
    a.nra4 = (l1.tile_tokens + 127) / 128;
  }
  a.bar = c->route_bar;
  a.status = c->status;
  a.timeout_ns = c->timeout_ns;
  const int grid = nch > c->num_sms ? nch : c->num_sms;  // one block per SM; the first nch own a chunk
  switch (topk_lane_candidates(g.n_experts)) {
    case 1: return launch_route_fused_p<1>(a, grid, s);
    case 2: return launch_route_fused_p<2>(a, grid, s);
    case 4: return launch_route_fused_p<4>(a, grid, s);
    case 8: return launch_route_fused_p<8>(a, grid, s);
    case 16: return launch_route_fused_p<16>(a, grid, s);
    default: return launch_route_fused_p<32>(a, grid, s);
  }
}

// NVFP4 forward: router, W_down and W_up in bf16; routed and shared experts as block-scaled FP4 GEMMs.
template <typename Mark>
cudaError_t forward_nvfp4(lmoe_ctx* c, const void* x, int T, void* y, int* idx, float* gate, cudaStream_t s,
                          Mark& mark, int& launches) {
  const lmoe_config& g = c->cfg;
  const int N = g.n_experts, K = g.top_k, d = g.d, l = g.latent, m = g.expert_ffn, ms = g.shared_ffn;
  const long long TK = (long long)T * K;
  const long long TKmax = (long long)g.max_tokens * K;
  const int vd = T <= 512 ? V_SMALL : V_LARGE;
  const int vg = TK <= 48LL * N ? V_SMALL4 : V_LARGE4;
  const bool split = vg == V_SMALL4;  // shared-expert GEMMs ride inside the expert launches
  const long long max_tiles4 = N + (TK + V_BN[vg] - 1) / V_BN[vg];  // token tiles of the expert launches
  unsigned* amax_x = reinterpret_cast<unsigned*>(c->work_counters + lmoe_ctx::kAmaxX);
  unsigned* amax_h = reinterpret_cast<unsigned*>(c->work_counters + lmoe_ctx::kAmaxH);
  float* g_x = c->act_g + 0;
  float* g_h = c->act_g + 1;
  const float* one = c->act_g + 2;
  cudaError_t e = cudaSuccess;
  auto chk = [&](cudaError_t r) {
    if (e == cudaSuccess) e = r;
  };
  auto grid_for = [&](long long work, int per_block) {
    long long b = (work + per_block - 1) / per_block;
    if (b > (long long)c->num_sms * 16) b = (long long)c->num_sms * 16;
    return (int)(b < 1 ? 1 : b);
  };

  // Decode sizes with the stacked router rows: the routing chain, the activation maxima, the x and h
  // quantisers and the grouped copy of h are one cooperative kernel
  const bool fused = vd == V_SMALL && vg == V_SMALL4 && c->fused_router && c->route_bar;
  const int nra = (V_BN[vg] + 127) / 128;  // scale row atoms per token tile of the FP4 variant
  const int sf_reps = vg == V_LARGE4 ? SF_WREP : 1;  // the prefill variant reads replicated scale atoms
  // 1. router logits and h = W_down x (bf16)
  int rks = 1;
  chk(router_stage(c, x, T, s, launches, fused, &rks));
  if (!mark(1)) return e;
  if (fused) {
    int ct;
    const int nch = n_chunks_for(T, N, &ct);
    UnitListSpec l1{c->units1, c->num_units, m, V_BN[vg], c->max_units1, c->unit_u0, V_TILE_M[vg]};
    UnitListSpec l2{c->units2, c->num_units + 1, l, V_BN[vg], c->max_units2, c->unit_u0 + N + 1, V_TILE_M[vg]};
    chk(launch_route_fused(c, T, rks, nch, ct, idx, gate, l1, l2, s, x));
    for (int i = 2; i <= 5; ++i)
      if (!mark(i)) return e;
  } else {
    // 2. quantise x (dynamic tensor scale); amax of h
    amax_act_kernel<<<grid_for((long long)T * d / 8, 256), 256, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16*>(x), (long long)T * d / 8, amax_x);
    quant_act_kernel<<<grid_for((long long)T * d / 16, 256), 256, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16*>(x), d, nullptr, T, T, nullptr, nullptr, N, V_BN[vg], nra, amax_x, c->xq,
        c->x_sf, g_x, c->status, sf_reps);
    amax_act_kernel<<<grid_for((long long)T * l / 8, 256), 256, 0, s>>>(c->h, (long long)T * l / 8, amax_h);
    chk(cudaGetLastError());
    if (!mark(2)) return e;
    // 3. top-K + softmax + per-chunk histogram
    int ct;
    const int nch = n_chunks_for(T, N, &ct);
    {
      const int parts = topk_parts(ct);
      if (parts > 1) chk(cudaMemsetAsync(c->chunk_counts, 0, (size_t)N * nch * sizeof(int), s));
      chk(launch_topk_hist(nch, parts, s, c->logits, c->b_router, T, N, K, ct, idx, gate, c->chunk_counts));
    }
    if (!mark(3)) return e;
    // 4. expert offsets and grouped-GEMM unit lists
    UnitListSpec l1{c->units1, c->num_units, m, V_BN[vg], c->max_units1, c->unit_u0, V_TILE_M[vg]};
    UnitListSpec l2{c->units2, c->num_units + 1, l, V_BN[vg], c->max_units2, c->unit_u0 + N + 1, V_TILE_M[vg]};
    scan_units_kernel<<<1, 1024, scan_smem_bytes(N, nch), s>>>(c->chunk_counts, nch, N, c->counts, c->offsets,
                                                                c->chunk_base, l1, l2, c->tile0, c->status);
    chk(cudaGetLastError());
    chk(launch_build_units(c, s, l1, l2, N));
    if (!mark(4)) return e;
    // 5. stable grouping; h quantised once per token, then its rows copied into grouped order with
    //    their scales in the expert GEMM's tile-local atoms
    assign_rows_kernel<<<nch, 32 * kAssignWarps, kAssignWarps * N * sizeof(int), s>>>(
        idx, gate, c->chunk_base, T, N, K, ct, c->row_of, c->tok_of_row, c->gate_of_row, c->status);
    quant_act_kernel<<<grid_for((long long)T * l / 16, 256), 256, 0, s>>>(c->h, l, nullptr, T, T, nullptr, nullptr, N,
                                                                           V_BN[vg], 0, amax_h, c->hq_tok, c->h_sf_tok,
                                                                           g_h, c->status, 1);
    {
      long long blocks = (TK + 7) / 8;  // one warp per row
      if (blocks > 16LL * c->num_sms) blocks = 16LL * c->num_sms;
      gather_act_q_kernel<<<(int)blocks, 256, 0, s>>>(c->hq_tok, c->h_sf_tok, l, c->tok_of_row, TK, T, c->offsets,
                                                       c->tile0, N, V_BN[vg], nra, c->hq, c->h_sf, c->status, sf_reps);
    }
    chk(cudaGetLastError());
    if (!mark(5)) return e;
  }
  // 6. expert up (FP4): u = NVFP4(sqrelu(W1_e h)); shared up u_s = NVFP4(sqrelu(W_s1 x))
  GemmProblem shared_up = problem4(d, EPI_SQRELU_NVFP4, c->usq, ms / 2, c->ws1_sf, c->wg + 2 * N, ms, c->x_sf, g_x);
  shared_up.out_sf = c->us_sf;
  shared_up.out_sf_stages = (ms + NVFP4_STAGE_K - 1) / NVFP4_STAGE_K;
  {
    GemmLaunch gl(c, vg, 4);
    if (split) gl.pre_dense(c->map_ws1q, c->map_xq[vg], shared_up, ms, T);
    GemmProblem p = problem4(l, EPI_SQRELU_NVFP4, c->uq, m / 2, c->w1_sf, c->wg, m, c->h_sf, g_h);
    p.out_sf = c->u_sf;
    p.out_sf_stages = (m + NVFP4_STAGE_K - 1) / NVFP4_STAGE_K;
    gl.main_grouped(c->map_w1q, c->map_hq[vg], p, c->units1, c->num_units, m, max_tiles4);
    chk(gl.run(s));
  }
  if (!split) {
    GemmLaunch gl(c, vg, 2);
    gl.main_dense(c->map_ws1q, c->map_xq[vg], shared_up, ms, T);
    chk(gl.run(s));
  }
  if (!mark(6)) return e;
  // 7. expert down (FP4) with the gate folded in: o = g * (W2_e u); y_s = W_s2 u_s (fp32)
  const GemmProblem shared_down = problem4(ms, EPI_F32, c->y_s, d, c->ws2_sf, c->wg + 2 * N + 1, d, c->us_sf, one);
  {
    GemmLaunch gl(c, vg, 5);
    if (split) gl.pre_dense(c->map_ws2q, c->map_usq[vg], shared_down, d, T);
    GemmProblem p = problem4(m, EPI_ROWSCALE_BF16, c->o, l, c->w2_sf, c->wg + N, l, c->u_sf, one);
    p.row_scale = c->gate_of_row;
    gl.main_grouped(c->map_w2q, c->map_uq[vg], p, c->units2, c->num_units + 1, l, max_tiles4);
    chk(gl.run(s));
  }
  if (!split) {
    GemmLaunch gl(c, vg, 3);
    gl.main_dense(c->map_ws2q, c->map_usq[vg], shared_down, d, T);
    chk(gl.run(s));
  }
  if (!mark(7)) return e;
  // 8. latent combine: zu[:, :l] = sum_k o[row_of[t, k]]
  chk(launch_combine(c->num_sms, s, c->o, c->row_of, T, K, l, c->zu, l + ms, TKmax, c->status));
  if (!mark(8)) return e;
  // 9. y = W_up z + y_s (bf16 GEMM)
  {
    GemmLaunch gl(c, vd, 6);
    GemmProblem p = problem(l, EPI_ADD_BF16, y, d);
    p.addend = c->y_s;
    p.ld_add = d;
    gl.main_dense(c->map_wup, c->map_z[vd], p, d, T);
    chk(gl.run(s));
  }
  if (!mark(9)) return e;
  launches += fused ? 5 : 13 + (split ? 0 : 2);
  return e;
}

// Host-buffer forwards of large bf16 batches run in chunks of kHostChunk tokens, so that the copy of
// one chunk's input and of another chunk's outputs overlap the layer's work on a third.  Each
// chunk still streams every expert's weights once, so chunks stay large (at 4096 tokens the layer
// is tensor-bound, not weight-bound).  NVFP4 layers are not chunked: their activation tensor
// scales are taken over the whole call's tokens.
constexpr int kHostChunk = 4096;

int host_chunk_tokens(const lmoe_ctx* c, int T) {
  if (c->nvfp4 || T < 2 * kHostChunk) return T;
  return kHostChunk;
}

// Chunk i: its input copy on host_in, its forward on s once that copy is done, its output copies on
// host_out once the forward is done.  The call forks from s (so the previous call's forward has
// finished reading x_dev before this call overwrites it) and joins back into s.
lmoe_status forward_host_chunked(lmoe_ctx* c, const void* x_host, int T, void* y_host, int* idx_host,
                                 float* gate_host, cudaStream_t s, int chunk) {
  const lmoe_config& g = c->cfg;
  const int n = (T + chunk - 1) / chunk;
  if (!c->host_in) {
    if (cudaStreamCreateWithFlags(&c->host_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&c->host_out, cudaStreamNonBlocking) != cudaSuccess)
      return LMOE_ERR_CUDA;
  }
  const size_t need = 2 * (size_t)n + 2;
  while (c->host_ev.size() < need) {
    cudaEvent_t e;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return LMOE_ERR_CUDA;
    c->host_ev.push_back(e);
  }
  cudaEvent_t* ev = c->host_ev.data();  // [0] fork, [1] join, [2 + 2i] input i copied, [3 + 2i] chunk i done
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  if (!ok(cudaEventRecord(ev[0], s)) || !ok(cudaStreamWaitEvent(c->host_in, ev[0], 0)) ||
      !ok(cudaStreamWaitEvent(c->host_out, ev[0], 0)))
    return LMOE_ERR_CUDA;
  const size_t row = (size_t)g.d * 2;
  lmoe_status st = LMOE_OK;
  for (int i = 0; i < n && st == LMOE_OK; ++i) {
    const size_t t0 = (size_t)i * chunk, tn = (size_t)(T - (int)t0 < chunk ? T - (int)t0 : chunk);
    if (!ok(cudaMemcpyAsync(reinterpret_cast<uint8_t*>(c->x_dev) + t0 * row,
                            reinterpret_cast<const uint8_t*>(x_host) + t0 * row, tn * row, cudaMemcpyHostToDevice,
                            c->host_in)) ||
        !ok(cudaEventRecord(ev[2 + 2 * i], c->host_in)))
      st = LMOE_ERR_CUDA;
  }
  for (int i = 0; i < n && st == LMOE_OK; ++i) {
    const size_t t0 = (size_t)i * chunk, tn = (size_t)(T - (int)t0 < chunk ? T - (int)t0 : chunk);
    const size_t k0 = t0 * g.top_k, kn = tn * g.top_k;
    if (!ok(cudaStreamWaitEvent(s, ev[2 + 2 * i], 0))) {
      st = LMOE_ERR_CUDA;
      break;
    }
    st = lmoe_forward(c, reinterpret_cast<uint8_t*>(c->x_dev) + t0 * row, (int)tn,
                      reinterpret_cast<uint8_t*>(c->y_dev) + t0 * row, c->idx_dev + k0, c->gate_dev + k0, s);
    if (st != LMOE_OK) break;
    if (!ok(cudaEventRecord(ev[3 + 2 * i], s)) || !ok(cudaStreamWaitEvent(c->host_out, ev[3 + 2 * i], 0)) ||
        !ok(cudaMemcpyAsync(reinterpret_cast<uint8_t*>(y_host) + t0 * row,
                            reinterpret_cast<const uint8_t*>(c->y_dev) + t0 * row, tn * row, cudaMemcpyDeviceToHost,
                            c->host_out)) ||
        (idx_host && !ok(cudaMemcpyAsync(idx_host + k0, c->idx_dev + k0, kn * 4, cudaMemcpyDeviceToHost, c->host_out))) ||
        (gate_host &&
         !ok(cudaMemcpyAsync(gate_host + k0, c->gate_dev + k0, kn * 4, cudaMemcpyDeviceToHost, c->host_out))))
      st = LMOE_ERR_CUDA;
  }
  // join both copy streams back into the caller's stream, on the error paths too, so that a
  // synchronisation of that stream covers every copy this call enqueued
  const bool joined = ok(cudaEventRecord(ev[1], c->host_in)) && ok(cudaStreamWaitEvent(s, ev[1], 0)) &&
                      ok(cudaEventRecord(ev[1], c->host_out)) && ok(cudaStreamWaitEvent(s, ev[1], 0));
  if (st == LMOE_OK && !joined) st = LMOE_ERR_CUDA;
  return st;
}

}  // namespace

extern "C" {

const char* lmoe_status_string(lmoe_status s) {
  switch (s) {
    case LMOE_OK: return "ok";
    case LMOE_ERR_INVALID_ARG: return "invalid argument";
    case LMOE_ERR_SHAPE: return "shape out of range";
    case LMOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case LMOE_ERR_OOM: return "device out of memory";
    case LMOE_ERR_CUDA: return "CUDA error";
    case LMOE_ERR_NOT_LOADED: return "weights not loaded";
    case LMOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case LMOE_ERR_DEVICE_INDEX: return "device-side index out of range";
    case LMOE_ERR_NO_DEVICE: return "no suitable CUDA device";
  }
  return "unknown status";
}

lmoe_status lmoe_create(const lmoe_config* cfg, int device, lmoe_handle* out) {
  if (!cfg || !out) return LMOE_ERR_INVALID_ARG;
  *out = nullptr;
  const lmoe_config& g = *cfg;
  if (g.d <= 0 || g.latent < 0 || g.n_experts <= 0 || g.top_k <= 0 || g.expert_ffn <= 0 || g.shared_ffn <= 0 ||
      g.max_tokens <= 0)
    return LMOE_ERR_INVALID_ARG;
  if (g.latent == 0 && g.precision != LMOE_PREC_BF16) return LMOE_ERR_UNSUPPORTED;
  if (g.precision != LMOE_PREC_BF16 && g.precision != LMOE_PREC_NVFP4) return LMOE_ERR_INVALID_ARG;
  if (g.weight_scale != LMOE_WSCALE_AMAX && g.weight_scale != LMOE_WSCALE_MSE) return LMOE_ERR_INVALID_ARG;
  if (g.d % 64 || g.latent % 64 || g.expert_ffn % 64 || g.shared_ffn % 64) return LMOE_ERR_UNSUPPORTED;
  if (g.n_experts > 1024 || g.n_experts % 16 || g.top_k > 32 || g.top_k > g.n_experts) return LMOE_ERR_UNSUPPORTED;
  if (g.precision == LMOE_PREC_NVFP4 &&
      (g.d % 128 || g.latent % 128 || g.expert_ffn % 128 || g.shared_ffn % 128))
    return LMOE_ERR_UNSUPPORTED;
  if (g.ep_world < 0 || (g.ep_world > 1 && (g.ep_rank < 0 || g.ep_rank >= g.ep_world))) return LMOE_ERR_INVALID_ARG;
  const bool ep = g.ep_world > 1;
  if (ep && (g.ep_world > EP_MAX_WORLD || g.n_experts % g.ep_world || g.precision != LMOE_PREC_BF16 ||
             g.latent == 0))
    return LMOE_ERR_UNSUPPORTED;
  const long long tk = (long long)g.max_tokens * g.top_k;
  // expert-side capacity: an expert-parallel rank may receive every rank's assignments
  const long long tk_exp = ep ? tk * g.ep_world : tk;
  if (tk_exp > 0x7fffffffLL / 2) return LMOE_ERR_UNSUPPORTED;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) return LMOE_ERR_NO_DEVICE;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess || prop.major != 10) return LMOE_ERR_NO_DEVICE;
  if (!load_encode()) return LMOE_ERR_CUDA;
  DeviceGuard dg(device);

  lmoe_ctx* c = new lmoe_ctx();
  c->cfg = g;
  c->device = device;
  c->num_sms = prop.multiProcessorCount;
  const int N = g.n_experts, K = g.top_k, d = g.d, l = g.latent, m = g.expert_ffn, ms = g.shared_ffn;
  const long long T = g.max_tokens;
  c->standard = l == 0;
  const int le = c->standard ? d : l;
  c->le = le;
  c->ep_world = ep ? g.ep_world : 0;
  c->ep_rank = ep ? g.ep_rank : 0;
  c->n_local = ep ? N / g.ep_world : N;
  c->tk_exp = tk_exp;
  const int NL = c->n_local;
  const int nft1 = (m + BLOCK_M - 1) / BLOCK_M, nft2 = (le + BLOCK_M - 1) / BLOCK_M;
  c->max_units1 = (int)(nft1 * (NL + (tk_exp + V_BN[V_SMALL] - 1) / V_BN[V_SMALL]));
  c->max_units2 = (int)(nft2 * (NL + (tk_exp + V_BN[V_SMALL] - 1) / V_BN[V_SMALL]));
  bool ok = true;
  ok = ok && dalloc(&c->logits, T * N) && dalloc(&c->idx, tk) && dalloc(&c->gate, tk);
  ok = ok && dalloc(&c->chunk_counts, 128LL * N) && dalloc(&c->chunk_base, 128LL * N);
  ok = ok && dalloc(&c->counts, N) && dalloc(&c->offsets, N + 1);
  ok = ok && dalloc(&c->row_of, tk_exp) && dalloc(&c->tok_of_row, tk_exp) && dalloc(&c->gate_of_row, tk_exp);
  if (!c->standard) ok = ok && dalloc(&c->h, T * l);
  ok = ok && dalloc(&c->h_perm, tk_exp * le) && dalloc(&c->u, tk_exp * m) && dalloc(&c->o, tk_exp * le);
  if (ep) {
    const int gp = g.top_k < g.ep_world ? g.top_k : g.ep_world;
    ok = ok && dalloc(&c->ep_ids, tk_exp) && dalloc(&c->ep_src, tk_exp) && dalloc(&c->ep_send_tok, T * gp);
  }
  ok = ok && dalloc(&c->zu, T * (l + ms));
  ok = ok && dalloc(&c->units1, c->max_units1) && dalloc(&c->units2, c->max_units2) && dalloc(&c->num_units, 2);
  ok = ok && dalloc(&c->status, 1) && dalloc(&c->work_counters, lmoe_ctx::kCounters) && dalloc(&c->route_bar, 2);
  ok = ok && dalloc(&c->tile0, N + 1) && dalloc(&c->unit_u0, 2 * (N + 1));
  {
    // router K-slice partials: stacked router + W_down rows at decode sizes, router rows otherwise
    const size_t small = (size_t)(T < lmoe_ctx::kSplitRows ? T : lmoe_ctx::kSplitRows) * (N + l);
    const size_t large = T > lmoe_ctx::kSplitRows ? (size_t)T * N : 0;
    ok = ok && dalloc(&c->router_part, (size_t)lmoe_ctx::kMaxSplits * (small > large ? small : large));
  }
  c->nvfp4 = g.precision == LMOE_PREC_NVFP4;
  // y_s = W_s2 u_s in fp32: needed at decode sizes (bf16) and at every size (NVFP4, standard MoE)
  ok = ok && dalloc(&c->y_s, (size_t)(c->nvfp4 || c->standard ? T : (T < 512 ? T : 512)) * d);
  if (c->nvfp4) {
    ok = ok && dalloc(&c->xq, T * d / 2) && dalloc(&c->x_sf, c->sf_bytes_dense(d));
    ok = ok && dalloc(&c->hq, tk * l / 2) && dalloc(&c->h_sf, c->sf_bytes_grouped(l));
    ok = ok && dalloc(&c->hq_tok, T * l / 2) && dalloc(&c->h_sf_tok, T * l / 16);
    ok = ok && dalloc(&c->uq, tk * m / 2) && dalloc(&c->u_sf, c->sf_bytes_grouped(m));
    ok = ok && dalloc(&c->usq, T * ms / 2) && dalloc(&c->us_sf, c->sf_bytes_dense(ms));
    ok = ok && dalloc(&c->act_g, 4);
  }
  if (!ok) {
    free_all(c);
    delete c;
    return LMOE_ERR_OOM;
  }
  cudaMemset(c->status, 0, sizeof(unsigned));
  cudaMemset(c->route_bar, 0, 2 * sizeof(unsigned));
  // rows that no expert writes must still be finite for the MMA (they are masked in the epilogue)
  cudaMemset(c->h_perm, 0, tk_exp * le * 2);
  cudaMemset(c->u, 0, tk_exp * m * 2);
  cudaMemset(c->zu, 0, T * (l + ms) * 2);
  for (int v = 0; v < 2; ++v) {
    ok = ok && make_map(&c->map_hperm[v], c->h_perm, tk_exp, le, le, V_BOXN[v]);
    if (v == V_LARGE) ok = ok && make_map(&c->map_hperm1, c->h_perm, tk_exp, le, le, V_BOXN[V_LARGE1]);
    ok = ok && make_map(&c->map_u[v], c->u, tk_exp, m, m, V_BOXN[v]);
    ok = ok && make_map(&c->map_zu[v], c->zu, T, l + ms, l + ms, V_BOXN[v]);
    if (!c->standard) ok = ok && make_map(&c->map_z[v], c->zu, T, l, l + ms, V_BOXN[v]);
    ok = ok && make_map(&c->map_us[v], c->zu + l, T, ms, l + ms, V_BOXN[v]);
  }
  ok = ok && cudaFuncSetAttribute(VT<V_SMALL>::fn(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  VT<V_SMALL>::smem()) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(VT<V_LARGE>::fn(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  VT<V_LARGE>::smem()) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(VT<V_SMALL4>::fn(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  VT<V_SMALL4>::smem()) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(VT<V_LARGE4>::fn(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  VT<V_LARGE4>::smem()) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(VT<V_LARGE1>::fn(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  VT<V_LARGE1>::smem()) == cudaSuccess;
  if (ok) {
    // a pair's two CTAs sit in one GPC: size the pair variant's grid to the pairs that fit at once
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(c->num_sms);
    cfg.blockDim = dim3(VT<V_LARGE>::THREADS);
    cfg.dynamicSmemBytes = VT<V_LARGE>::smem();
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, VT<V_LARGE>::fn(), &cfg) != cudaSuccess || nc < 1) {
      cudaGetLastError();
      nc = c->num_sms / 2;
    }
    c->pair_workers = nc < c->num_sms / 2 ? nc : c->num_sms / 2;
  }
  if (ok && c->nvfp4) {
    // scale padding (beyond K / 16) must read as zero; stale rows must hold finite scales
    cudaMemset(c->x_sf, 0, c->sf_bytes_dense(d));
    cudaMemset(c->h_sf, 0, c->sf_bytes_grouped(l));
    cudaMemset(c->u_sf, 0, c->sf_bytes_grouped(m));
    cudaMemset(c->us_sf, 0, c->sf_bytes_dense(ms));
    cudaMemset(c->xq, 0, T * d / 2);
    cudaMemset(c->hq, 0, tk * l / 2);
    cudaMemset(c->uq, 0, tk * m / 2);
    cudaMemset(c->usq, 0, T * ms / 2);
    const float one[4] = {1.f, 1.f, 1.f, 1.f};
    ok = cudaMemcpy(c->act_g, one, sizeof(one), cudaMemcpyHostToDevice) == cudaSuccess;
    for (int v = V_SMALL4; v <= V_LARGE4; ++v) {
      ok = ok && make_map_u8(&c->map_xq[v], c->xq, T, d / 2, d / 2, V_BOXN[v]);
      ok = ok && make_map_u8(&c->map_hq[v], c->hq, tk, l / 2, l / 2, V_BOXN[v]);
      ok = ok && make_map_u8(&c->map_uq[v], c->uq, tk, m / 2, m / 2, V_BOXN[v]);
      ok = ok && make_map_u8(&c->map_usq[v], c->usq, T, ms / 2, ms / 2, V_BOXN[v]);
    }
  }
  ok = ok && cudaFuncSetAttribute(reinterpret_cast<const void*>(scan_units_kernel),
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, kScanSmemMax) == cudaSuccess;
  {
    // the attribute belongs to the kernel, not to this handle: size it for the largest N any handle
    // may have, so that creating a layer never lowers another layer's limit
    const int rsm = (int)route_fused_smem(1024, kRouteFusedThreads / 32);
    const void* rk[] = {reinterpret_cast<const void*>(route_fused_kernel<1>),
                        reinterpret_cast<const void*>(route_fused_kernel<2>),
                        reinterpret_cast<const void*>(route_fused_kernel<4>),
                        reinterpret_cast<const void*>(route_fused_kernel<8>),
                        reinterpret_cast<const void*>(route_fused_kernel<16>),
                        reinterpret_cast<const void*>(route_fused_kernel<32>)};
    for (const void* f : rk)
      ok = ok && cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, rsm) == cudaSuccess;
  }
  if (!ok || cudaDeviceSynchronize() != cudaSuccess) {
    free_all(c);
    delete c;
    return LMOE_ERR_CUDA;
  }
  (void)d;
  *out = c;
  return LMOE_OK;
}

lmoe_status lmoe_load_weights(lmoe_handle c, const lmoe_weights* w, void* stream) {
  if (!c || !w) return LMOE_ERR_INVALID_ARG;
  if (!w->w_router || !w->w1 || !w->w2 || !w->ws1 || !w->ws2) return LMOE_ERR_INVALID_ARG;
  // a standard MoE has no projections; a LatentMoE layer needs both
  if (c->standard ? (w->w_down || w->w_up) : (!w->w_down || !w->w_up)) return LMOE_ERR_INVALID_ARG;
  if (w->dtype != LMOE_DTYPE_BF16 && w->dtype != LMOE_DTYPE_F32) return LMOE_ERR_INVALID_ARG;
  if (c->cfg.has_router_bias && !w->b_router) return LMOE_ERR_INVALID_ARG;
  const void* ptrs[] = {w->w_router, w->w_down, w->w_up, w->w1, w->w2, w->ws1, w->ws2};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return LMOE_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const lmoe_config& g = c->cfg;
  const int N = g.n_experts, d = g.d, l = g.latent, m = g.expert_ffn, ms = g.shared_ffn;
  const int le = c->le;
  const int f32 = w->dtype == LMOE_DTYPE_F32;

  // release weights of a previous load
  void* old[] = {c->w_rd,  c->w_r32, c->w_down, c->b_router, c->w_cat,  c->ws1,  c->w1,    c->w2,
                 c->w1q,   c->w2q,   c->ws1q,   c->ws2q,     c->w1_sf,  c->w2_sf, c->ws1_sf, c->ws2_sf,
                 c->wg,    c->w_amax};
  cudaStreamSynchronize(s);
  for (void* p : old)
    if (p) cudaFree(p);
  c->w_rd = nullptr;
  c->w_r32 = nullptr;
  c->w_down = nullptr;
  c->b_router = nullptr;
  c->w_cat = nullptr;
  c->ws1 = c->w1 = c->w2 = nullptr;
  c->w1q = c->w2q = c->ws1q = c->ws2q = nullptr;
  c->w1_sf = c->w2_sf = c->ws1_sf = c->ws2_sf = nullptr;
  c->wg = nullptr;
  c->w_amax = nullptr;
  c->loaded = false;

  c->router_f32 = f32;
  c->fused_router = !f32 && (N % BLOCK_M == 0) && !c->standard;
  bool ok = true;
  auto conv = [&](const void* src, long long rows, int cols, long long src_ld, __nv_bfloat16* dst, long long dst_ld,
                  int col0) {
    const long long total = rows * cols;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 4 * 148 * 8) blocks = 4 * 148 * 8;
    convert_2d_kernel<<<blocks, 256, 0, s>>>(src, f32, rows, cols, src_ld, dst, dst_ld, col0);
    return cudaGetLastError() == cudaSuccess;
  };
  if (c->router_f32) {
    ok = ok && dalloc(&c->w_r32, (size_t)N * d) &&
         cudaMemcpyAsync(c->w_r32, w->w_router, (size_t)N * d * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (!c->standard) ok = ok && dalloc(&c->w_down, (size_t)l * d) && conv(w->w_down, l, d, d, c->w_down, d, 0);
  } else if (c->fused_router) {
    ok = ok && dalloc(&c->w_rd, (size_t)(N + l) * d);
    ok = ok && conv(w->w_router, N, d, d, c->w_rd, d, 0) && conv(w->w_down, l, d, d, c->w_rd + (size_t)N * d, d, 0);
  } else {
    ok = ok && dalloc(&c->w_rd, (size_t)N * d) && conv(w->w_router, N, d, d, c->w_rd, d, 0);
    if (!c->standard) ok = ok && dalloc(&c->w_down, (size_t)l * d) && conv(w->w_down, l, d, d, c->w_down, d, 0);
  }
  if (g.has_router_bias)
    ok = ok && dalloc(&c->b_router, N) &&
         cudaMemcpyAsync(c->b_router, w->b_router, (size_t)N * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
  ok = ok && dalloc(&c->w_cat, (size_t)d * (l + ms));
  if (!c->standard) ok = ok && conv(w->w_up, d, l, l, c->w_cat, l + ms, 0);
  ok = ok && conv(w->ws2, d, ms, ms, c->w_cat, l + ms, l);
  ok = ok && dalloc(&c->ws1, (size_t)ms * d) && conv(w->ws1, ms, d, d, c->ws1, d, 0);
  const int NL = c->n_local;  // the experts this handle holds
  ok = ok && dalloc(&c->w1, (size_t)NL * m * le) && conv(w->w1, (long long)NL * m, le, le, c->w1, le, 0);
  ok = ok && dalloc(&c->w2, (size_t)NL * le * m) && conv(w->w2, (long long)NL * le, m, m, c->w2, m, 0);
  if (!ok) return LMOE_ERR_OOM;
  if (c->nvfp4) {
    // quantise W1, W2, W_s1, W_s2 on the device; keep only codes, scale atoms and tensor scales
    __nv_bfloat16* ws2_tmp = nullptr;
    ok = ok && dalloc(&ws2_tmp, (size_t)d * ms) && conv(w->ws2, d, ms, ms, ws2_tmp, ms, 0);
    auto sf_bytes = [](long long rows, int K) {
      return (size_t)(rows / 128) * sf_atoms_k(K) * SF_ATOM_BYTES * SF_WREP;
    };
    ok = ok && dalloc(&c->w1q, (size_t)N * m * l / 2) && dalloc(&c->w1_sf, sf_bytes((long long)N * m, l));
    ok = ok && dalloc(&c->w2q, (size_t)N * l * m / 2) && dalloc(&c->w2_sf, sf_bytes((long long)N * l, m));
    ok = ok && dalloc(&c->ws1q, (size_t)ms * d / 2) && dalloc(&c->ws1_sf, sf_bytes(ms, d));
    ok = ok && dalloc(&c->ws2q, (size_t)d * ms / 2) && dalloc(&c->ws2_sf, sf_bytes(d, ms));
    ok = ok && dalloc(&c->wg, 2 * N + 2) && dalloc(&c->w_amax, 2 * N + 2);
    if (!ok) {
      if (ws2_tmp) cudaFree(ws2_tmp);
      return LMOE_ERR_OOM;
    }
    ok = cudaMemsetAsync(c->w_amax, 0, (2 * N + 2) * sizeof(unsigned), s) == cudaSuccess;
    ok = ok && cudaMemsetAsync(c->w1_sf, 0, sf_bytes((long long)N * m, l), s) == cudaSuccess;
    ok = ok && cudaMemsetAsync(c->w2_sf, 0, sf_bytes((long long)N * l, m), s) == cudaSuccess;
    ok = ok && cudaMemsetAsync(c->ws1_sf, 0, sf_bytes(ms, d), s) == cudaSuccess;
    ok = ok && cudaMemsetAsync(c->ws2_sf, 0, sf_bytes(d, ms), s) == cudaSuccess;
    struct Q {
      const __nv_bfloat16* src;
      long long rows;
      int K;
      long long rows_per_g;
      int groups;
      uint8_t* codes;
      uint8_t* sf;
      int g0;
    } qs[4] = {{c->w1, (long long)N * m, l, m, N, c->w1q, c->w1_sf, 0},
               {c->w2, (long long)N * l, m, l, N, c->w2q, c->w2_sf, N},
               {c->ws1, ms, d, ms, 1, c->ws1q, c->ws1_sf, 2 * N},
               {ws2_tmp, d, ms, d, 1, c->ws2q, c->ws2_sf, 2 * N + 1}};
    for (const Q& q : qs) {
      amax_groups_kernel<<<dim3(16, q.groups), 256, 0, s>>>(q.src, q.rows_per_g * q.K, c->w_amax + q.g0);
      const long long blocks_needed = (q.rows * (q.K / 16) + 255) / 256;
      const int blocks = (int)(blocks_needed < 148LL * 64 ? blocks_needed : 148LL * 64);
      quant_weight_kernel<<<blocks, 256, 0, s>>>(q.src, q.rows, q.K, q.rows_per_g, c->w_amax + q.g0, q.codes, q.sf,
                                                 c->wg + q.g0, c->cfg.weight_scale == LMOE_WSCALE_MSE);
    }
    ok = ok && cudaGetLastError() == cudaSuccess && cudaStreamSynchronize(s) == cudaSuccess;
    cudaFree(ws2_tmp);
    cudaFree(c->w1);
    cudaFree(c->w2);
    cudaFree(c->ws1);
    c->w1 = c->w2 = c->ws1 = nullptr;
    ok = ok && make_map_u8(&c->map_w1q, c->w1q, (uint64_t)N * m, l / 2, l / 2, BLOCK_M);
    ok = ok && make_map_u8(&c->map_w2q, c->w2q, (uint64_t)N * l, m / 2, m / 2, BLOCK_M);
    ok = ok && make_map_u8(&c->map_ws1q, c->ws1q, ms, d / 2, d / 2, BLOCK_M);
    ok = ok && make_map_u8(&c->map_ws2q, c->ws2q, d, ms / 2, ms / 2, BLOCK_M);
    if (!ok) return LMOE_ERR_CUDA;
  }
  // map_r / map_down: the router and W_down rows alone (views of the stacked matrix when fused)
  if (c->fused_router) ok = ok && make_map(&c->map_rd, c->w_rd, N + l, d, d, BLOCK_M);
  if (!c->router_f32) ok = ok && make_map(&c->map_r, c->w_rd, N, d, d, BLOCK_M);
  if (!c->standard)
    ok = ok && make_map(&c->map_down, c->fused_router ? c->w_rd + (size_t)N * d : c->w_down, l, d, d, BLOCK_M);
  ok = ok && make_map(&c->map_cat, c->w_cat, d, l + ms, l + ms, BLOCK_M);
  if (!c->standard) ok = ok && make_map(&c->map_wup, c->w_cat, d, l, l + ms, BLOCK_M);
  ok = ok && make_map(&c->map_ws2, c->w_cat + l, d, ms, l + ms, BLOCK_M);
  if (!c->nvfp4) {
    ok = ok && make_map(&c->map_ws1, c->ws1, ms, d, d, BLOCK_M);
    ok = ok && make_map(&c->map_w1, c->w1, (uint64_t)NL * m, le, le, BLOCK_M);
    ok = ok && make_map(&c->map_w2, c->w2, (uint64_t)NL * le, m, m, BLOCK_M);
  }
  if (!ok) return LMOE_ERR_CUDA;
  c->loaded = true;
  return LMOE_OK;
}

lmoe_status lmoe_forward(lmoe_handle c, const void* x, int32_t T, void* y, int32_t* topk_idx, float* topk_gate,
                         void* stream) {
  if (!c) return LMOE_ERR_INVALID_ARG;
  if (T < 0 || T > c->cfg.max_tokens) return LMOE_ERR_SHAPE;
  if (!c->loaded) return LMOE_ERR_NOT_LOADED;
  if (c->ep_world > 1) return LMOE_ERR_UNSUPPORTED;  // an expert-parallel rank runs the lmoe_ep_* steps
  if (T == 0) return LMOE_OK;
  if (!x || !y) return LMOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || (topk_idx && !aligned16(topk_idx)) || (topk_gate && !aligned16(topk_gate)))
    return LMOE_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const lmoe_config& g = c->cfg;
  const int N = g.n_experts, K = g.top_k, d = g.d, l = g.latent, m = g.expert_ffn, ms = g.shared_ffn;
  const int le = c->le;  // expert input / output width: l, or d for a standard MoE
  const long long TK = (long long)T * K;
  const long long TKmax = (long long)g.max_tokens * K;
  const int vd = T <= 512 ? V_SMALL : V_LARGE;
  const int vg = TK <= 48LL * N ? V_SMALL : V_LARGE;

  if (!set_x_maps(c, x, T)) return LMOE_ERR_CUDA;
  int* idx = topk_idx ? topk_idx : c->idx;
  float* gate = topk_gate ? topk_gate : c->gate;
  cudaError_t e = cudaSuccess;
  auto chk = [&](cudaError_t r) {
    if (e == cudaSuccess) e = r;
  };
  const bool prof = c->prof_on && c->prof_n < lmoe_ctx::kProfMax;
  cudaEvent_t* ev = prof ? &c->prof_ev[(size_t)c->prof_n * (LMOE_NUM_STAGES + 1)] : nullptr;
  // stage boundary: record the profiling event; false once any launch has failed, so that no later
  // kernel runs on routing state a failed launch did not write
  auto mark = [&](int i) {
    if (prof) chk(cudaEventRecord(ev[i], s));
    return e == cudaSuccess;
  };
  int launches = 0;
  // Decode sizes with the stacked router rows (bf16): the routing chain is one cooperative kernel,
  // which also zeroes the unit counters of the launches after it
  const bool fused_route = !c->nvfp4 && c->fused_router && vd == V_SMALL && vg == V_SMALL && c->route_bar;
  if (!fused_route) chk(cudaMemsetAsync(c->work_counters, 0, lmoe_ctx::kCounters * sizeof(int), s));
  if (!mark(0)) return cuda_status(e);
  if (c->nvfp4) {
    const cudaError_t r = forward_nvfp4(c, x, T, y, idx, gate, s, mark, launches);
    chk(r);
    c->launches = launches;
    if (prof) ++c->prof_n;
    c->last_T = T;
    return cuda_status(e);
  }

  // At decode sizes (T <= 512 with decode-sized expert groups) the shared expert's two matrices ride
  // inside the expert launches as dense pre problems, and the output GEMM only does W_up z + y_s.
  const bool split = vd == V_SMALL && vg == V_SMALL && c->y_s != nullptr;

  // 1. router logits and the latent h = W_down x (with the fused routing kernel: the router GEMM's
  //    K-slice partials, summed by that kernel)
  int rks = 1;
  chk(router_stage(c, x, T, s, launches, fused_route, &rks));
  if (!mark(1)) return cuda_status(e);
  // 2. shared expert, first matrix: zu[:, l:] = sqrelu(W_s1 x)   (inside the expert-up launch when split)
  const GemmProblem shared_up = problem(d, EPI_SQRELU_BF16, c->zu, l + ms, l);
  if (!split) {
    GemmLaunch g(c, vd, 3);
    g.main_dense(c->map_ws1, c->map_x[vd], shared_up, ms, T);
    chk(g.run(s));
    launches += 1;
  }
  if (!mark(2)) return cuda_status(e);
  int ct;
  const int nch = n_chunks_for(T, N, &ct);
  // the expert-up GEMM's variant.  With at least a full token tile per expert on average (prefill),
  // the single-CTA one (same token tile as the pair), which has no half-empty pair tiles at 2688
  // features; with fewer (skewed loads: most experts hold one partial tile and stream their weights),
  // the pair, whose deeper ring keeps more weight bytes in flight (measured: 0.79 vs 0.85 ms there)
  const int vu = (vg == V_LARGE && TK >= (long long)V_BN[V_LARGE1] * N) ? V_LARGE1 : vg;
  UnitListSpec l1{c->units1, c->num_units, m, V_BN[vu], c->max_units1, c->unit_u0, V_TILE_M[vu]};
  UnitListSpec l2{c->units2, c->num_units + 1, le, V_BN[vg], c->max_units2, c->unit_u0 + N + 1, V_TILE_M[vg]};
  if (fused_route) {
    // 3-5. slice sum, top-K, expert scan, unit lists, stable rows and gather in one launch
    chk(launch_route_fused(c, T, rks, nch, ct, idx, gate, l1, l2, s));
    if (!mark(3)) return cuda_status(e);
    if (!mark(4)) return cuda_status(e);
    if (!mark(5)) return cuda_status(e);
  } else {
    // 3. top-K + softmax + per-chunk histogram
    {
      const int parts = topk_parts(ct);
      if (parts > 1) chk(cudaMemsetAsync(c->chunk_counts, 0, (size_t)N * nch * sizeof(int), s));
      chk(launch_topk_hist(nch, parts, s, c->logits, c->b_router, T, N, K, ct, idx, gate, c->chunk_counts));
    }
    if (!mark(3)) return cuda_status(e);
    // 4. expert offsets and grouped-GEMM unit lists
    scan_units_kernel<<<1, 1024, scan_smem_bytes(N, nch), s>>>(c->chunk_counts, nch, N, c->counts, c->offsets,
                                                                c->chunk_base, l1, l2, c->tile0, c->status);
    chk(cudaGetLastError());
    chk(launch_build_units(c, s, l1, l2, N));
    if (!mark(4)) return cuda_status(e);
    // 5. stable grouping, then the gather of latent rows into grouped order
    assign_rows_kernel<<<nch, 32 * kAssignWarps, kAssignWarps * N * sizeof(int), s>>>(
        idx, gate, c->chunk_base, T, N, K, ct, c->row_of, c->tok_of_row, c->gate_of_row, c->status);
    chk(cudaGetLastError());
    {
      long long warps = (TK + GATHER_ROWS - 1) / GATHER_ROWS;
      long long blocks = (warps + 7) / 8;
      if (blocks > (long long)c->num_sms * 8) blocks = (long long)c->num_sms * 8;
      // a standard MoE's experts read x itself
      const __nv_bfloat16* src = c->standard ? reinterpret_cast<const __nv_bfloat16*>(x) : c->h;
      gather_rows_kernel<<<(int)blocks, 256, 0, s>>>(src, c->tok_of_row, TK, T, le, c->h_perm, c->status);
      chk(cudaGetLastError());
    }
    if (!mark(5)) return cuda_status(e);
  }
  // 6. expert up: u = sqrelu(W1_e h)
  {
    GemmLaunch g(c, vu, 4);
    if (split) g.pre_dense(c->map_ws1, c->map_x[vd], shared_up, ms, T);
    g.main_grouped(c->map_w1, vu == V_LARGE1 ? c->map_hperm1 : c->map_hperm[vg], problem(le, EPI_SQRELU_BF16, c->u, m),
                   c->units1, c->num_units, m, 0);
    chk(g.run(s));
  }
  if (!mark(6)) return cuda_status(e);
  // 7. expert down with the gate folded in: o = g * (W2_e u); when split, also y_s = W_s2 u_s (fp32)
  {
    GemmLaunch g(c, vg, 5);
    if (split) g.pre_dense(c->map_ws2, c->map_us[vd], problem(ms, EPI_F32, c->y_s, d), d, T);
    GemmProblem p = problem(m, EPI_ROWSCALE_BF16, c->o, le);
    p.row_scale = c->gate_of_row;
    g.main_grouped(c->map_w2, c->map_u[vg], p, c->units2, c->num_units + 1, le, 0);
    chk(g.run(s));
  }
  if (c->standard && !split) {
    // a standard MoE adds the shared expert after the combine: y_s = W_s2 u_s (fp32)
    GemmLaunch g(c, vd, 6);
    g.main_dense(c->map_ws2, c->map_us[vd], problem(ms, EPI_F32, c->y_s, d), d, T);
    chk(g.run(s));
    launches += 1;
  }
  if (!mark(7)) return cuda_status(e);
  // 8. latent combine: zu[:, :l] = sum_k o[row_of[t, k]]; a standard MoE's combine writes
  //    y = sum_k o[row_of[t, k]] + y_s and the layer ends here
  if (c->standard)
    chk(launch_combine(c->num_sms, s, c->o, c->row_of, T, K, d, reinterpret_cast<__nv_bfloat16*>(y), d, TKmax,
                       c->status, c->y_s, d));
  else
    chk(launch_combine(c->num_sms, s, c->o, c->row_of, T, K, l, c->zu, l + ms, TKmax, c->status));
  if (!mark(8)) return cuda_status(e);
  if (c->standard) {
    if (!mark(9)) return cuda_status(e);
    launches += 8;
    c->launches = launches;
    if (prof) ++c->prof_n;
    c->last_T = T;
    return cuda_status(e);
  }
  // 9. y = [z | sqrelu(W_s1 x)] [W_up | W_s2]^T, or y = W_up z + y_s when split
  {
    GemmLaunch g(c, vd, 6);
    if (split) {
      GemmProblem p = problem(l, EPI_ADD_BF16, y, d);
      p.addend = c->y_s;
      p.ld_add = d;
      g.main_dense(c->map_wup, c->map_z[vd], p, d, T);
    } else {
      g.main_dense(c->map_cat, c->map_zu[vd], problem(l + ms, EPI_BF16, y, d), d, T);
    }
    chk(g.run(s));
  }
  if (!mark(9)) return cuda_status(e);
  launches += fused_route ? 5 : 9;
  c->launches = launches;
  if (prof) ++c->prof_n;
  c->last_T = T;
  (void)TK;
  return cuda_status(e);
}

lmoe_status lmoe_forward_host(lmoe_handle c, const void* x_host, int32_t T, void* y_host, int32_t* idx_host,
                              float* gate_host, void* stream) {
  if (!c) return LMOE_ERR_INVALID_ARG;
  if (T < 0 || T > c->cfg.max_tokens) return LMOE_ERR_SHAPE;
  if (!c->loaded) return LMOE_ERR_NOT_LOADED;
  if (T == 0) return LMOE_OK;
  if (!x_host || !y_host) return LMOE_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  const lmoe_config& g = c->cfg;
  const size_t xb = (size_t)g.max_tokens * g.d * 2, kb = (size_t)g.max_tokens * g.top_k;
  if (!c->x_dev) {
    if (!dalloc(&c->x_dev, xb / 2) || !dalloc(&c->y_dev, xb / 2) || !dalloc(&c->idx_dev, kb) ||
        !dalloc(&c->gate_dev, kb))
      return LMOE_ERR_OOM;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int chunk = host_chunk_tokens(c, T);
  if (chunk < T) return forward_host_chunked(c, x_host, T, y_host, idx_host, gate_host, s, chunk);
  const size_t bytes = (size_t)T * g.d * 2;
  if (cudaMemcpyAsync(c->x_dev, x_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) return LMOE_ERR_CUDA;
  lmoe_status st = lmoe_forward(c, c->x_dev, T, c->y_dev, c->idx_dev, c->gate_dev, stream);
  if (st != LMOE_OK) return st;
  if (cudaMemcpyAsync(y_host, c->y_dev, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) return LMOE_ERR_CUDA;
  const size_t ib = (size_t)T * g.top_k * 4;
  if (idx_host && cudaMemcpyAsync(idx_host, c->idx_dev, ib, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return LMOE_ERR_CUDA;
  if (gate_host && cudaMemcpyAsync(gate_host, c->gate_dev, ib, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return LMOE_ERR_CUDA;
  return LMOE_OK;
}

// ---------------------------------------------------------------------------------------- expert parallelism
lmoe_status lmoe_ep_dispatch(lmoe_handle c, const void* x, int32_t T, int32_t* topk_idx, float* topk_gate,
                             void* send_rows, int32_t* send_meta, float* send_gate, int32_t* counts,
                             int32_t* tok_pairs, void* stream) {
  if (!c) return LMOE_ERR_INVALID_ARG;
  if (c->ep_world < 2) return LMOE_ERR_UNSUPPORTED;
  if (T < 0 || T > c->cfg.max_tokens) return LMOE_ERR_SHAPE;
  if (!c->loaded) return LMOE_ERR_NOT_LOADED;
  if (T == 0) return LMOE_OK;
  const void* ptrs[] = {x, topk_idx, topk_gate, send_rows, send_meta, send_gate, counts, tok_pairs};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LMOE_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const lmoe_config& g = c->cfg;
  const int N = g.n_experts, K = g.top_k, G = c->ep_world;
  const int GP = K < G ? K : G;
  if (!set_x_maps(c, x, T)) return LMOE_ERR_CUDA;
  cudaError_t e = cudaMemsetAsync(c->work_counters, 0, lmoe_ctx::kCounters * sizeof(int), s);
  int launches = 0;
  if (e == cudaSuccess) e = router_stage(c, x, T, s, launches);
  int ct;
  const int nch = n_chunks_for(T, N, &ct);
  const int parts = topk_parts(ct);
  if (e == cudaSuccess && parts > 1) e = cudaMemsetAsync(c->chunk_counts, 0, (size_t)N * nch * sizeof(int), s);
  if (e == cudaSuccess)
    e = launch_topk_hist(nch, parts, s, c->logits, c->b_router, T, N, K, ct, topk_idx, topk_gate, c->chunk_counts);
  if (e == cudaSuccess) {
    ep_plan_kernel<<<1, EP_PLAN_THREADS, 0, s>>>(topk_idx, topk_gate, T, K, N, N / G, G, GP, counts, c->ep_send_tok,
                                                 send_meta, send_gate, tok_pairs, c->status);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) {
    long long blocks = ((long long)T * GP + 7) / 8;  // one warp per row
    if (blocks > 8LL * c->num_sms) blocks = 8LL * c->num_sms;
    ep_gather_send_kernel<<<(int)blocks, 256, 0, s>>>(c->h, c->ep_send_tok, counts, G, T, g.latent,
                                                      reinterpret_cast<__nv_bfloat16*>(send_rows), c->status);
    e = cudaGetLastError();
  }
  c->last_T = T;
  return cuda_status(e);
}

lmoe_status lmoe_ep_experts(lmoe_handle c, const void* recv_rows, int32_t R, const int32_t* recv_meta,
                            const float* recv_gate, int32_t A, float* partial, void* stream) {
  if (!c) return LMOE_ERR_INVALID_ARG;
  if (c->ep_world < 2) return LMOE_ERR_UNSUPPORTED;
  if (!c->loaded) return LMOE_ERR_NOT_LOADED;
  const lmoe_config& g = c->cfg;
  const int K = g.top_k, G = c->ep_world, l = g.latent, m = g.expert_ffn, NL = c->n_local;
  const long long GP = K < G ? K : G;
  if (R < 0 || A < 0 || (long long)R > (long long)G * g.max_tokens * GP || A > c->tk_exp) return LMOE_ERR_SHAPE;
  if (R == 0) return LMOE_OK;
  if (!recv_rows || !partial || !aligned16(recv_rows) || !aligned16(partial)) return LMOE_ERR_INVALID_ARG;
  if (A > 0 && (!recv_meta || !recv_gate || !aligned16(recv_meta) || !aligned16(recv_gate)))
    return LMOE_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (A == 0) return cuda_status(cudaMemsetAsync(partial, 0, (size_t)R * l * sizeof(float), s));
  cudaError_t e = cudaMemsetAsync(c->work_counters, 0, lmoe_ctx::kCounters * sizeof(int), s);
  auto chk = [&](cudaError_t r) {
    if (e == cudaSuccess) e = r;
    return e == cudaSuccess;
  };
  // the received assignments, grouped stably (arrival order) by local expert: the single-GPU
  // dispatch kernels with the assignments as "tokens" of one slot each
  ep_split_meta_kernel<<<(int)((A + 255) / 256 < 4 * c->num_sms ? (A + 255) / 256 : 4 * c->num_sms), 256, 0, s>>>(
      recv_meta, A, c->ep_ids, c->ep_src);
  if (!chk(cudaGetLastError())) return cuda_status(e);
  int ct;
  const int nch = n_chunks_for(A, NL, &ct);
  ids_hist_kernel<<<nch, 256, NL * sizeof(int), s>>>(c->ep_ids, A, NL, ct, c->chunk_counts);
  if (!chk(cudaGetLastError())) return cuda_status(e);
  const int vg = A <= 48LL * NL ? V_SMALL : V_LARGE;
  UnitListSpec l1{c->units1, c->num_units, m, V_BN[vg], c->max_units1, c->unit_u0, V_TILE_M[vg]};
  UnitListSpec l2{c->units2, c->num_units + 1, l, V_BN[vg], c->max_units2, c->unit_u0 + g.n_experts + 1,
                  V_TILE_M[vg]};
  scan_units_kernel<<<1, 1024, scan_smem_bytes(NL, nch), s>>>(c->chunk_counts, nch, NL, c->counts, c->offsets,
                                                               c->chunk_base, l1, l2, c->tile0, c->status);
  if (!chk(cudaGetLastError()) || !chk(launch_build_units(c, s, l1, l2, NL))) return cuda_status(e);
  assign_rows_kernel<<<nch, 32 * kAssignWarps, kAssignWarps * NL * sizeof(int), s>>>(
      c->ep_ids, recv_gate, c->chunk_base, A, NL, 1, ct, c->row_of, c->tok_of_row, c->gate_of_row, c->status);
  if (!chk(cudaGetLastError())) return cuda_status(e);
  {
    long long blocks = ((long long)A + 7) / 8;  // one warp per grouped row
    if (blocks > 8LL * c->num_sms) blocks = 8LL * c->num_sms;
    gather_src_kernel<<<(int)blocks, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(recv_rows), R, c->ep_src,
                                                  c->tok_of_row, A, A, l, c->h_perm, c->status);
    if (!chk(cudaGetLastError())) return cuda_status(e);
  }
  // the owned experts, gate folded into the second GEMM
  {
    GemmLaunch gl(c, vg, 4);
    gl.main_grouped(c->map_w1, c->map_hperm[vg], problem(l, EPI_SQRELU_BF16, c->u, m), c->units1, c->num_units, m, 0);
    if (!chk(gl.run(s))) return cuda_status(e);
  }
  {
    GemmLaunch gl(c, vg, 5);
    GemmProblem p = problem(m, EPI_ROWSCALE_BF16, c->o, l);
    p.row_scale = c->gate_of_row;
    gl.main_grouped(c->map_w2, c->map_u[vg], p, c->units2, c->num_units + 1, l, 0);
    if (!chk(gl.run(s))) return cuda_status(e);
  }
  // one fp32 partial latent sum per received row
  {
    long long blocks = ((long long)R * (l / 8) + 255) / 256;
    if (blocks > 8LL * c->num_sms) blocks = 8LL * c->num_sms;
    ep_pair_reduce_kernel<<<(int)blocks, 256, 0, s>>>(c->o, c->row_of, c->ep_src, A, A, R, l, partial, c->status);
    chk(cudaGetLastError());
  }
  return cuda_status(e);
}

lmoe_status lmoe_ep_combine(lmoe_handle c, const void* x, int32_t T, const float* back, const int32_t* tok_pairs,
                            void* y, void* stream) {
  if (!c) return LMOE_ERR_INVALID_ARG;
  if (c->ep_world < 2) return LMOE_ERR_UNSUPPORTED;
  if (T < 0 || T > c->cfg.max_tokens) return LMOE_ERR_SHAPE;
  if (!c->loaded) return LMOE_ERR_NOT_LOADED;
  if (T == 0) return LMOE_OK;
  const void* ptrs[] = {x, back, tok_pairs, y};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LMOE_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const lmoe_config& g = c->cfg;
  const int K = g.top_k, G = c->ep_world, d = g.d, l = g.latent, ms = g.shared_ffn;
  const int GP = K < G ? K : G;
  const int vd = T <= 512 ? V_SMALL : V_LARGE;
  if (!set_x_maps(c, x, T)) return LMOE_ERR_CUDA;
  cudaError_t e = cudaMemsetAsync(c->work_counters, 0, lmoe_ctx::kCounters * sizeof(int), s);
  if (e == cudaSuccess) {
    // z = the token's partial sums in ascending owner order, into zu[:, :l]
    long long blocks = ((long long)T * (l / 8) + 255) / 256;
    if (blocks > 8LL * c->num_sms) blocks = 8LL * c->num_sms;
    ep_combine_kernel<<<(int)blocks, 256, 0, s>>>(back, T * GP, tok_pairs, T, GP, l, c->zu, l + ms, c->status);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) {
    // shared expert, first matrix: zu[:, l:] = sqrelu(W_s1 x)
    GemmLaunch gl(c, vd, 3);
    gl.main_dense(c->map_ws1, c->map_x[vd], problem(d, EPI_SQRELU_BF16, c->zu, l + ms, l), ms, T);
    e = gl.run(s);
  }
  if (e == cudaSuccess) {
    // y = [z | sqrelu(W_s1 x)] [W_up | W_s2]^T
    GemmLaunch gl(c, vd, 6);
    gl.main_dense(c->map_cat, c->map_zu[vd], problem(l + ms, EPI_BF16, y, d), d, T);
    e = gl.run(s);
  }
  return cuda_status(e);
}

lmoe_status lmoe_export_nvfp4(lmoe_handle c, int32_t which, int32_t index, uint8_t* codes_host, uint8_t* scales_host,
                              float* gscale_host) {
  if (!c || !codes_host || !scales_host || !gscale_host) return LMOE_ERR_INVALID_ARG;
  if (!c->nvfp4) return LMOE_ERR_UNSUPPORTED;
  if (!c->loaded) return LMOE_ERR_NOT_LOADED;
  const lmoe_config& g = c->cfg;
  const int N = g.n_experts, d = g.d, l = g.latent, m = g.expert_ffn, ms = g.shared_ffn;
  const uint8_t* codes = nullptr;
  const uint8_t* atoms = nullptr;
  long long row0 = 0, rows = 0;
  int K = 0, gi = 0;
  switch (which) {
    case 0:
      if (index < 0 || index >= N) return LMOE_ERR_SHAPE;
      codes = c->w1q, atoms = c->w1_sf, row0 = (long long)index * m, rows = m, K = l, gi = index;
      break;
    case 1:
      if (index < 0 || index >= N) return LMOE_ERR_SHAPE;
      codes = c->w2q, atoms = c->w2_sf, row0 = (long long)index * l, rows = l, K = m, gi = N + index;
      break;
    case 2: codes = c->ws1q, atoms = c->ws1_sf, rows = ms, K = d, gi = 2 * N; break;
    case 3: codes = c->ws2q, atoms = c->ws2_sf, rows = d, K = ms, gi = 2 * N + 1; break;
    default: return LMOE_ERR_SHAPE;
  }
  DeviceGuard dg(c->device);
  if (cudaDeviceSynchronize() != cudaSuccess) return LMOE_ERR_CUDA;
  if (cudaMemcpy(codes_host, codes + row0 * (K / 2), (size_t)rows * (K / 2), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LMOE_ERR_CUDA;
  if (cudaMemcpy(gscale_host, c->wg + gi, sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess) return LMOE_ERR_CUDA;
  // the matrix's scale atoms are contiguous (its rows start on a 128-row tile)
  const int atoms_k = sf_atoms_k(K);
  const size_t atom_bytes = (size_t)(rows / 128) * atoms_k * SF_ATOM_BYTES * SF_WREP;
  std::vector<uint8_t> tmp(atom_bytes);
  if (cudaMemcpy(tmp.data(), atoms + (row0 / 128) * atoms_k * SF_ATOM_BYTES * SF_WREP, atom_bytes,
                 cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return LMOE_ERR_CUDA;
  for (long long r = 0; r < rows; ++r)
    for (int kb = 0; kb < K / 16; ++kb) scales_host[r * (K / 16) + kb] = tmp[sf_atom_offset(r, kb, atoms_k)];
  return LMOE_OK;
}

// One thread waits on a shared-memory mbarrier whose single expected arrival never comes.
__global__ void wait_timeout_probe_kernel(unsigned* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns)) atomicOr(status, DEV_STATUS_TIMEOUT);
}

lmoe_status lmoe_selftest_wait_timeout(lmoe_handle c, uint64_t limit_ns, void* stream) {
  if (!c) return LMOE_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  const unsigned long long lim = std::min<uint64_t>(std::max<uint64_t>(limit_ns, 1000ull), 2000000000ull);
  wait_timeout_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(c->status, lim);
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

lmoe_status lmoe_get_device_status(lmoe_handle c) {
  if (!c) return LMOE_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  if (cudaDeviceSynchronize() != cudaSuccess) return LMOE_ERR_CUDA;
  unsigned st = 0;
  if (cudaMemcpy(&st, c->status, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return LMOE_ERR_CUDA;
  cudaMemset(c->status, 0, sizeof(unsigned));
  // a bounded wait that gave up may have left the routing kernel's grid barrier mid-phase
  if (st & DEV_STATUS_TIMEOUT) cudaMemset(c->route_bar, 0, 2 * sizeof(unsigned));
  if (st & DEV_STATUS_TIMEOUT) return LMOE_ERR_DEVICE_TIMEOUT;
  if (st & DEV_STATUS_BAD_INDEX) return LMOE_ERR_DEVICE_INDEX;
  return LMOE_OK;
}

lmoe_status lmoe_inspect(lmoe_handle c, int32_t which, void** dev_ptr, int64_t* count) {
  if (!c || !dev_ptr || !count) return LMOE_ERR_INVALID_ARG;
  if (which >= LMOE_BUF_XQ && !c->nvfp4 && which != LMOE_BUF_Y_S) return LMOE_ERR_UNSUPPORTED;
  const lmoe_config& g = c->cfg;
  const long long T = c->last_T, TK = T * g.top_k;
  switch (which) {
    case LMOE_BUF_LOGITS: *dev_ptr = c->logits; *count = T * g.n_experts; break;
    case LMOE_BUF_COUNTS: *dev_ptr = c->counts; *count = g.n_experts; break;
    case LMOE_BUF_OFFSETS: *dev_ptr = c->offsets; *count = g.n_experts + 1; break;
    case LMOE_BUF_ROW_OF: *dev_ptr = c->row_of; *count = TK; break;
    case LMOE_BUF_TOK_OF_ROW: *dev_ptr = c->tok_of_row; *count = TK; break;
    case LMOE_BUF_H:
      if (c->standard) return LMOE_ERR_UNSUPPORTED;
      *dev_ptr = c->h;
      *count = T * g.latent;
      break;
    case LMOE_BUF_Z: *dev_ptr = c->zu; *count = T * (g.latent + g.shared_ffn); break;
    case LMOE_BUF_U: *dev_ptr = c->u; *count = TK * g.expert_ffn; break;
    case LMOE_BUF_XQ: *dev_ptr = c->xq; *count = T * g.d / 2; break;
    case LMOE_BUF_X_SF: *dev_ptr = c->x_sf; *count = (int64_t)c->sf_bytes_dense(g.d); break;
    case LMOE_BUF_HQ: *dev_ptr = c->hq; *count = TK * g.latent / 2; break;
    case LMOE_BUF_H_SF: *dev_ptr = c->h_sf; *count = (int64_t)c->sf_bytes_grouped(g.latent); break;
    case LMOE_BUF_UQ: *dev_ptr = c->uq; *count = TK * g.expert_ffn / 2; break;
    case LMOE_BUF_U_SF: *dev_ptr = c->u_sf; *count = (int64_t)c->sf_bytes_grouped(g.expert_ffn); break;
    case LMOE_BUF_USQ: *dev_ptr = c->usq; *count = T * g.shared_ffn / 2; break;
    case LMOE_BUF_US_SF: *dev_ptr = c->us_sf; *count = (int64_t)c->sf_bytes_dense(g.shared_ffn); break;
    case LMOE_BUF_Y_S: *dev_ptr = c->y_s; *count = T * g.d; break;
    case LMOE_BUF_ACT_SCALE: *dev_ptr = c->act_g; *count = 2; break;
    default: return LMOE_ERR_INVALID_ARG;
  }
  return LMOE_OK;
}

lmoe_status lmoe_profile(lmoe_handle c, int32_t enable) {
  if (!c) return LMOE_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  if (enable && c->prof_ev.empty()) {
    c->prof_ev.resize((size_t)lmoe_ctx::kProfMax * (LMOE_NUM_STAGES + 1));
    for (auto& e : c->prof_ev)
      if (cudaEventCreate(&e) != cudaSuccess) return LMOE_ERR_CUDA;
  }
  if (enable) c->prof_n = 0;
  c->prof_on = enable != 0;
  return LMOE_OK;
}

lmoe_status lmoe_profile_read(lmoe_handle c, double* stage_ms, int32_t* forwards, int32_t* launches) {
  if (!c || !stage_ms) return LMOE_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  for (int i = 0; i < LMOE_NUM_STAGES; ++i) stage_ms[i] = 0.0;
  for (int f = 0; f < c->prof_n; ++f) {
    cudaEvent_t* ev = &c->prof_ev[(size_t)f * (LMOE_NUM_STAGES + 1)];
    if (cudaEventSynchronize(ev[LMOE_NUM_STAGES]) != cudaSuccess) return LMOE_ERR_CUDA;
    for (int i = 0; i < LMOE_NUM_STAGES; ++i) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, ev[i], ev[i + 1]) != cudaSuccess) return LMOE_ERR_CUDA;
      stage_ms[i] += ms;
    }
  }
  if (forwards) *forwards = c->prof_n;
  if (launches) *launches = c->launches;
  return LMOE_OK;
}

void lmoe_destroy(lmoe_handle c) {
  if (!c) return;
  {
    DeviceGuard dg(c->device);
    cudaDeviceSynchronize();
    for (auto& e : c->prof_ev) cudaEventDestroy(e);
    for (auto& e : c->host_ev) cudaEventDestroy(e);
    if (c->host_in) cudaStreamDestroy(c->host_in);
    if (c->host_out) cudaStreamDestroy(c->host_out);
    free_all(c);
  }
  delete c;
}

}  // extern "C"
// ------------------------------------------------------------------------------------------------
// Routing without device allocation.  Its scratch (per-chunk expert histograms and bases, and the
// grouped-row maps the scatter kernel writes) lives in this file-scope device array.  Host code must
// not pass the array's name to a kernel (on the host it is only a stand-in symbol); the device
// address is looked up once per device with cudaGetSymbolAddress.
// ------------------------------------------------------------------------------------------------
constexpr int kNoAllocMaxExperts = 1024;
constexpr int kNoAllocMaxChunks = 128;                 // n_chunks_for() never exceeds this
constexpr long long kNoAllocMaxAssignments = 131072;   // T * K
constexpr size_t kNoAllocChunkWords = (size_t)kNoAllocMaxExperts * kNoAllocMaxChunks;
constexpr size_t kNoAllocWords = 2 * kNoAllocChunkWords + 2 * (size_t)kNoAllocMaxAssignments + 64;

static __device__ __align__(256) unsigned int g_noalloc_scratch[kNoAllocWords];

namespace {
std::mutex g_noalloc_mu;
constexpr int kNoAllocMaxDevices = 64;
unsigned int* g_noalloc_addr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up on first use).
cudaError_t noalloc_scratch(unsigned int** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(scan_units_kernel),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kScanSmemMax);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = static_cast<unsigned int*>(p);
  }
  *out = g_noalloc_addr[dev];
  return cudaSuccess;
}
}  // namespace

extern "C" lmoe_status lmoe_route_noalloc(const float* logits, const float* bias, int32_t T, int32_t n_experts,
                                          int32_t top_k, int32_t* topk_idx, float* topk_gate, int32_t* counts,
                                          int32_t* offsets, int32_t* row_of, uint32_t* status_dev, void* stream) {
  const int N = n_experts, K = top_k;
  if (N < 1 || N > kNoAllocMaxExperts || K < 1 || K > 32 || K > N) return LMOE_ERR_UNSUPPORTED;
  if (T < 0 || (long long)T * K > kNoAllocMaxAssignments) return LMOE_ERR_SHAPE;
  if (T == 0) return LMOE_OK;
  if (!logits || !topk_idx || !topk_gate || !counts || !offsets || !row_of) return LMOE_ERR_INVALID_ARG;
  if (!aligned16(logits) || (bias && !aligned16(bias)) || !aligned16(topk_idx) || !aligned16(topk_gate) ||
      !aligned16(counts) || !aligned16(offsets) || !aligned16(row_of) ||
      (status_dev && (reinterpret_cast<uintptr_t>(status_dev) & 3u)))
    return LMOE_ERR_INVALID_ARG;
  unsigned int* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return LMOE_ERR_CUDA;
  int* chunk_counts = reinterpret_cast<int*>(scratch);
  int* chunk_base = chunk_counts + kNoAllocChunkWords;
  int* tok_of_row = chunk_base + kNoAllocChunkWords;
  float* gate_of_row = reinterpret_cast<float*>(tok_of_row + kNoAllocMaxAssignments);
  // the kernels raise status bits in the caller's word when one is given, else in a scratch word
  // that nobody reads
  unsigned* status = status_dev ? status_dev : reinterpret_cast<unsigned*>(gate_of_row + kNoAllocMaxAssignments);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the status word accumulates with atomicOr, so it must start at zero; every other scratch word
  // is fully written before it is read
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), s) != cudaSuccess) return LMOE_ERR_CUDA;
  int ct;
  const int nch = n_chunks_for(T, N, &ct);
  if (launch_topk_hist(nch, 1, s, logits, bias, T, N, K, ct, topk_idx, topk_gate, chunk_counts) !=
      cudaSuccess)
    return LMOE_ERR_CUDA;
  UnitListSpec none{nullptr, nullptr, 0, 64, 0, nullptr, BLOCK_M};
  scan_units_kernel<<<1, 1024, scan_smem_bytes(N, nch), s>>>(chunk_counts, nch, N, counts, offsets, chunk_base,
                                                              none, none, nullptr, status);
  if (cudaGetLastError() != cudaSuccess) return LMOE_ERR_CUDA;
  assign_rows_kernel<<<nch, 32, N * sizeof(int), s>>>(topk_idx, topk_gate, chunk_base, T, N, K, ct, row_of,
                                                     tok_of_row, gate_of_row, status);
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}
