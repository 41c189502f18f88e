// Persistent, warp-specialised tcgen05 GEMM used for every contraction of the LatentMoE layer.
//
//   out[tok, f] = epi( sum_k W[f, k] * act[tok, k] )
//
// W (weights, K-major) is the MMA's A operand: 128 output features per tile fill the M = 128 rows of
// the tensor core.  The activations (K-major) are the B operand: up to BN_MAX tokens per tile form N,
// rounded up to a multiple of 16.  With tokens on N, an expert that holds only ~11 tokens (the
// T = 256 decode batch spread over 512 experts) costs an N = 16 MMA instead of a 128-row tile that is
// 90 % padding, and every expert weight byte is streamed exactly once per token tile.
//
// Two operand formats (template flag FP4):
//   bf16   kind::f16, 64 elements (128 bytes) of K per pipeline stage
//   NVFP4  kind::mxf4nvf4 with 16-element E4M3 block scales, 256 E2M1 elements (128 bytes) of K per
//          stage.  Scales arrive by bulk copy in 512-byte atoms and the MMA issuer moves them into
//          TMEM with tcgen05.cp: weight atoms are stored replicated (two 128x256b copies per stage);
//          the decode variant keeps a token tile's activation scales resident in TMEM across the
//          tile's units (copied by its first unit), the prefill variant reads replicated activation
//          atoms (one 128x256b copy per K atom).  The epilogue multiplies by the two fp32 tensor
//          scales.
//
// Roles (64 + 32 * EPIW threads; EPIW = 4 epilogue warps, or 8 for the NVFP4 prefill variant):
//   warp 0      producer: streams W and activation tiles (TMA) and scales into a STAGES-deep ring,
//               and publishes each unit's descriptor to the other roles through a shared-memory ring
//   warp 1      MMA issuer: allocates TMEM, one lane issues tcgen05 MMAs into one of two TMEM
//               accumulators (double buffered, so the epilogue of tile i overlaps the MMAs of i+1)
//   warps 2..   epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes 32*(w%4)..),
//               elementwise op, transpose through shared memory, vector stores
//
// Work units are (weight row block, token block) pairs.  Dense GEMMs enumerate them from the
// launch arguments; the grouped expert GEMMs read a unit list that the routing kernels built on the
// device, so no host round trip sits between routing and the experts.  One launch can carry two
// problems: an optional dense "pre" problem whose units come first, then the main problem.  At
// decode sizes every problem is a weight stream, so folding a small dense GEMM into an expert launch
// costs only its bytes instead of a launch that cannot fill the GPU.
#pragma once
#include <cuda_bf16.h>

#include "nvfp4.cuh"
#include "ptx.cuh"

namespace lmoe {

enum EpiKind : int {
  EPI_BF16 = 0,           // out = bf16(acc)
  EPI_F32 = 1,            // out = acc (fp32)
  EPI_SQRELU_BF16 = 2,    // out = bf16(max(acc, 0)^2)
  EPI_ROWSCALE_BF16 = 3,  // out = bf16(acc * row_scale[token row])
  EPI_ADD_BF16 = 5,       // out = bf16(acc + addend[token row, f])  (fp32 addend)
  EPI_SQRELU_NVFP4 = 6,   // out = NVFP4(max(acc, 0)^2) with tensor scale 1: codes to out, scales to out_sf
};

// One unit of GEMM work.  a_row: first W row of the tile; b_row: first activation row (also the
// output row); f0: first output feature (column) of the tile; nm = n_valid | (m_valid << 16) with
// n_valid tokens (1..BN_MAX) and m_valid features (1..128, a multiple of 16; a multiple of 32 for
// EPI_SQRELU_NVFP4); tile: token-tile id (NVFP4 activation scales are stored per token tile).
struct GemmUnit {
  int a_row, b_row, f0, nm;
  int tile, kslice, pad1, pad2;  // kslice: K slice of a split dense unit (0 otherwise); in the
                                 // kernel's unit ring pad1 = problem, pad2 = unit (-1: no more units)
};

// One GEMM problem of a launch: K extent, epilogue, NVFP4 scales, and (for dense problems) the grid.
struct GemmProblem {
  int num_k_blocks;           // pipeline stages along K (64 bf16 or 256 FP4 elements each)
  int epi;
  void* out;
  long long ldo;              // output row pitch (elements; bytes for EPI_SQRELU_NVFP4 codes)
  int out_col0;               // output column offset
  const float* row_scale;     // EPI_ROWSCALE_BF16
  const float* addend;        // EPI_ADD_BF16
  long long ld_add;
  uint8_t* out_sf;            // EPI_SQRELU_NVFP4 scales, tile-local atoms (act_sf_offset)
  int out_sf_stages;          // 256-element stages of the output's K
  int weights_streamed;       // 1: every weight tile is read by one unit only (L2 evict-first)
  // NVFP4 operands
  const uint8_t* w_sf;        // weight scale atoms
  int w_atoms_k;              // K atoms per 128-row tile
  const float* w_gscale;      // per-group weight tensor scale, group = a_row / w_rows_per_g
  int w_rows_per_g;
  const uint8_t* act_sf;      // activation scales, tile-local atoms (act_sf_offset)
  int act_sf_stages;          // 256-element stages of the activations' K
  const float* act_gscale;    // activation tensor scale (device scalar)
  int sfb_resident;           // 1: a token tile's activation scales for the whole K are loaded once
                              // and stay in TMEM while consecutive units use the same tile
  // dense enumeration
  int dense_ftiles;           // feature tiles
  int dense_ttiles;           // token tiles (fastest-varying unit index)
  int dense_feat;             // output features (rows of W)
  int dense_tokens;           // tokens (rows of act)
  // split K (dense bf16 problems with EPI_F32): k_splits slices of the K blocks, slice s writes its
  // fp32 partial at out + s * split_stride; the caller sums the slices
  int k_splits;
  long long split_stride;
};

struct GemmArgs {
  GemmProblem prob[2];        // [0] main problem, [1] optional dense pre problem (tensor maps *_1)
  int n_pre_units;            // units of prob[1], enumerated first
  int main_dense_units;       // units of prob[0] when it is dense (units == nullptr)
  const GemmUnit* units;      // prob[0] grouped: device unit list
  const int* num_units;       // prob[0] grouped: device unit count
  int dynamic;                // 1: claims come from work_counter; 0: CTA c takes claims c, c + grid, ...
  int chunk;                  // main-problem units per claim (>= 1); every pre unit is a claim of its own
  int* work_counter;          // zero before a dynamic launch
  unsigned* status;           // device status word
  unsigned long long timeout_ns;
};

constexpr int GEMM_THREADS = 192;  // producer warp, MMA warp and four epilogue warps (the default)
constexpr int UNIT_RING = 4;
constexpr int BLOCK_M = 128;
constexpr int BLOCK_K = 64;                 // bf16 elements per stage (one 128-byte swizzle row)
constexpr int A_STAGE_BYTES = BLOCK_M * 128;
constexpr int EPI_STAGE_BYTES = 32 * 32 * 4;  // per epilogue warp: 32 tokens x 32 features fp32
constexpr int SF_ATOM_BYTES = 512;

// RES_STAGES > 0 (FP4): room for the activation scales of one token tile over up to RES_STAGES
// K stages, kept in TMEM across consecutive units of that tile (problems with sfb_resident): the
// tile's first unit loads and copies them stage by stage, its later units reuse them.
// PAIR: the CTA is one of a pair sharing cta_group::2 MMAs (M = 256); it holds half of the token
// tile's rows per stage.
template <int BN_MAX, int STAGES, bool FP4, int ACC_SPLIT, int RES_STAGES, bool PAIR = false, int EPIW = 4>
struct GemmSmem {
  static constexpr int NRA = (BN_MAX + 127) / 128;                    // 128-row scale atoms of B
  static constexpr int B_STAGE_BYTES = (PAIR ? BN_MAX / 2 : BN_MAX) * 128;
  static constexpr int SFA_STAGE_BYTES = FP4 ? 4 * SF_ATOM_BYTES * SF_WREP : 0;  // replicated weight atoms
  // activation scales of the variants without resident scales (prefill sizes) are stored replicated
  // like the weight scales, so one 128x256b copy moves both 128-row atoms of a K atom
  static constexpr int SFB_REP = (FP4 && RES_STAGES == 0) ? SF_WREP : 1;
  static_assert(SFB_REP == 1 || NRA == 2, "replicated activation scales pair the two row atoms of a K atom");
  static constexpr int SFB_STAGE_BYTES = FP4 ? 4 * NRA * SF_ATOM_BYTES * SFB_REP : 0;
  static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES + SFA_STAGE_BYTES + SFB_STAGE_BYTES;
  static constexpr int EPI_OFF = STAGES * STAGE_BYTES;
  static constexpr int BAR_OFF = EPI_OFF + EPIW * EPI_STAGE_BYTES;
  static constexpr int BYTES = BAR_OFF + 512;
  // barrier block: 2 * STAGES + 21 mbarriers, TMEM slot and abort flag, unit ring, claim mailbox
  static_assert(16 * STAGES + 176 + 32 * UNIT_RING + 4 * UNIT_RING <= 512, "barrier block overflows");
  static constexpr int ALLOC = BYTES + 1024;  // slack for 1024-byte alignment of the base
  // TMEM: two accumulator buffers (double buffering), each ACC_SPLIT partial fp32 accumulators of
  // BN_MAX columns; then (FP4) SF_SLOTS rotating slots of weight scales (SFA: 4 MMAs x 4 columns per
  // stage), then the activation scales (SFB): either SF_SLOTS rotating per-stage slots (4 MMAs x NRA
  // x 4 columns) or one resident tile of up to RES_STAGES stages, sharing the same columns.  Every
  // MMA's scale address is 4-column aligned (the block-scaled MMA faults on a misaligned scale
  // address).
  static constexpr int ACC_COLS = ACC_SPLIT * BN_MAX;
  static constexpr int SF_COL0 = 2 * ACC_COLS;
  static constexpr int sf_need(int slots) {
    return 16 * slots + 16 * NRA * (RES_STAGES > slots ? RES_STAGES : slots);
  }
  static constexpr int SF_SLOTS = !FP4 ? 1
                                  : SF_COL0 + sf_need(4) <= 512 ? 4
                                  : SF_COL0 + sf_need(3) <= 512 ? 3
                                  : SF_COL0 + sf_need(2) <= 512 ? 2
                                                                : 1;
  static constexpr int SFA_COL0 = SF_COL0;
  static constexpr int SFB_COL0 = SF_COL0 + 16 * SF_SLOTS;
  static constexpr int TMEM_NEED = SF_COL0 + (FP4 ? sf_need(SF_SLOTS) : 0);
  static constexpr uint32_t TMEM_COLS = (TMEM_NEED <= 32)    ? 32
                                        : (TMEM_NEED <= 64)  ? 64
                                        : (TMEM_NEED <= 128) ? 128
                                        : (TMEM_NEED <= 256) ? 256
                                                             : 512;
  static_assert(TMEM_NEED <= 512 && SF_SLOTS >= 1, "TMEM holds 512 columns");
  static_assert(ALLOC <= 232448, "shared memory per CTA");
};

template <int BN_MAX, int TILE_M>
__device__ __forceinline__ GemmUnit dense_unit(const GemmProblem& p, int u) {
  GemmUnit r;
  // K slices outermost; token tiles of one weight tile run on adjacent CTAs, so the weight tile is
  // read from HBM once
  const int per_slice = p.dense_ftiles * p.dense_ttiles;
  const int ks = p.k_splits > 1 ? u / per_slice : 0;
  u -= ks * per_slice;
  r.kslice = ks;
  const int tt = u % p.dense_ttiles;
  const int ft = u / p.dense_ttiles;
  r.a_row = ft * TILE_M;
  r.f0 = r.a_row;
  r.b_row = tt * BN_MAX;
  const int mv = min(TILE_M, p.dense_feat - r.f0);
  const int nv = min(BN_MAX, p.dense_tokens - r.b_row);
  r.nm = nv | (mv << 16);
  r.tile = tt;
  return r;
}

// K blocks [kb0, kb1) of a unit: all of them, or its slice of a split problem.
__device__ __forceinline__ void unit_k_range(const GemmProblem& p, const GemmUnit& un, int& kb0, int& kb1) {
  if (p.k_splits > 1) {
    const int per = (p.num_k_blocks + p.k_splits - 1) / p.k_splits;
    kb0 = un.kslice * per;
    kb1 = min(p.num_k_blocks, kb0 + per);
  } else {
    kb0 = 0;
    kb1 = p.num_k_blocks;
  }
}

// Global unit u of the launch: which problem it belongs to, and its tile.  The pre problem's units
// come first (measured: spreading them through the expert units was slower at decode sizes).
// In a CTA pair a unit covers 256 weight rows; each CTA of the pair sees its own 128 (unit_at
// returns the CTA's half: rows and first feature shifted by 128 * rank, valid features clamped).
template <int BN_MAX, int TILE_M>
__device__ __forceinline__ GemmUnit unit_at(const GemmArgs& a, int u, int& pid, uint32_t pair_rank = 0) {
  GemmUnit r;
  if (u < a.n_pre_units) {
    pid = 1;
    r = dense_unit<BN_MAX, TILE_M>(a.prob[1], u);
  } else {
    pid = 0;
    u -= a.n_pre_units;
    r = (a.units != nullptr) ? a.units[u] : dense_unit<BN_MAX, TILE_M>(a.prob[0], u);
  }
  if (TILE_M > BLOCK_M) {
    const int sh = BLOCK_M * (int)pair_rank;
    r.a_row += sh;
    r.f0 += sh;
    const int mv = max(0, min(BLOCK_M, (r.nm >> 16) - sh));
    r.nm = (r.nm & 0xFFFF) | (mv << 16);
  }
  return r;
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float v) {
  __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&b);
}

// ACC_SPLIT > 1: consecutive MMAs of a tile rotate over ACC_SPLIT independent partial accumulators,
// summed by the epilogue.  With few tokens (N = 16..64) one MMA is far shorter than the tensor pipe's
// latency, and MMAs chained on one accumulator would each wait for the previous one.
//
// PAIR (bf16 only): the grid is made of clusters of two CTAs that share cta_group::2 MMAs of
// M = 256 weight rows.  Each CTA loads its own 128 weight rows and half of the token tile (the even
// CTA tokens 0..N/2-1, the odd one N/2..N-1) into its shared memory; the even CTA's producer expects
// both halves' bytes on its stage barrier, its MMA issuer runs the pair's MMAs and commits them to
// both CTAs' barriers, and each CTA's epilogue drains its own half of the accumulator from its own
// TMEM.  Per stage an SM then reads 32 KB for 128 x 256 x 64 MACs instead of 48 KB.  Both CTAs
// walk the same unit sequence: static claims by pair, or dynamic claims taken by the even CTA and
// passed to the odd one through a mailbox in its shared memory.
//
// EPIW epilogue warps (4 or 8): with 8, two warps share each TMEM lane quadrant and take alternate
// 32-token chunks of a tile (for epilogues that cost more than the tile's MMAs, such as the NVFP4
// quantisation of u after short-K units).
template <int BN_MAX, int STAGES, int BOXN, bool FP4, int ACC_SPLIT, int RES_STAGES, bool PAIR, int EPIW>
__global__ void __launch_bounds__(64 + 32 * EPIW, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap map_w0, const __grid_constant__ CUtensorMap map_act0,
                   const __grid_constant__ CUtensorMap map_w1, const __grid_constant__ CUtensorMap map_act1,
                   const GemmArgs args) {
  using S = GemmSmem<BN_MAX, STAGES, FP4, ACC_SPLIT, RES_STAGES, PAIR, EPIW>;
  static_assert(EPIW == 4 || EPIW == 8, "one or two epilogue warps per TMEM lane quadrant");
  constexpr int TILE_M = PAIR ? 2 * BLOCK_M : BLOCK_M;
  static_assert(BN_MAX % BOXN == 0 && BOXN % 8 == 0, "token box must tile the token block");
  static_assert(BN_MAX % 16 == 0 && BN_MAX <= 256, "MMA N limit");
  static_assert(!PAIR || (!FP4 && ACC_SPLIT == 1 && BOXN == BN_MAX / 2), "pair variant: bf16, one box per half");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* ufull = drain + 1;              // unit ring: producer -> MMA issuer and epilogue warps
  uint64_t* uempty = ufull + UNIT_RING;
  uint64_t* mfull = uempty + UNIT_RING;     // claim mailbox (pair, dynamic): even -> odd CTA
  uint64_t* mempty = mfull + UNIT_RING;     //   odd -> even CTA (the slot may be rewritten)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mempty + UNIT_RING);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // unit ring entries: the producer publishes each unit's whole descriptor (16-byte aligned: the
  // barrier block is 16 * STAGES + 176 bytes long), so the MMA issuer and the epilogue start a unit
  // without a global-memory round trip
  int4* unit_ring = reinterpret_cast<int4*>(tmem_slot + 2);
  volatile int* mailbox = reinterpret_cast<volatile int*>(unit_ring + 2 * UNIT_RING);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t prank = PAIR ? cluster_ctarank() : 0u;  // rank in the pair; 0 issues the MMAs
  const bool issuer = prank == 0;
  // the next launch may begin (its CTAs take SMs as this grid's CTAs exit)
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], PAIR ? 2 * EPIW : EPIW);  // a pair's issuer waits for both CTAs' epilogue warps
    }
    mbar_init(drain, 1);
    for (int i = 0; i < UNIT_RING; ++i) {
      mbar_init(&ufull[i], 1);
      mbar_init(&uempty[i], 1 + EPIW);  // the MMA issuer and the epilogue warps
      mbar_init(&mfull[i], 1);
      mbar_init(&mempty[i], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_w0);
    tma_prefetch_desc(&map_act0);
    if (args.n_pre_units > 0) {
      tma_prefetch_desc(&map_w1);
      tma_prefetch_desc(&map_act1);
    }
  }
  if (warp == 1) {
    if constexpr (PAIR) tmem_alloc_pair(tmem_slot, S::TMEM_COLS);
    else tmem_alloc(tmem_slot, S::TMEM_COLS);
  }
  tc_fence_before();
  __syncthreads();
  // a pair's barriers and TMEM are set up on both sides before either CTA signals the other
  if constexpr (PAIR) cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // everything above is this CTA's own set-up; from here on the kernel reads what earlier launches
  // wrote (unit lists, activations, scales, addends)
  griddep_wait();

  const int num_units = args.n_pre_units + ((args.units != nullptr) ? *args.num_units : args.main_dense_units);
  // Every role walks the same sequence of units, published by the producer through the unit ring
  // (a negative entry ends the sequence).
  const uint64_t tmo = args.timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer (one lane)
    if (lane == 0) {
      const uint64_t pol_first = policy_evict_first();
      const uint64_t pol_normal = policy_evict_normal();
      const uint64_t pol_a = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      int uslot = 0;
      uint32_t uphase = 0;
      // Work is handed out in claims: claim c < n_pre is pre unit c; later claims cover `chunk`
      // consecutive main units each (consecutive main units share a token tile, feature tiles
      // fastest).  Dynamic launches take the next claim from work_counter one unit ahead, so the
      // atomic's round trip overlaps the loads; static launches take claims c, c + grid, ...
      const int n_pre = args.n_pre_units;
      const int chunk = args.chunk > 0 ? args.chunk : 1;
      const int n_claims = n_pre + (num_units - n_pre + chunk - 1) / chunk;
      // a pair is one worker: claims by pair index, or the even CTA's dynamic claims forwarded
      const int worker = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
      const int n_workers = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
      int mslot = 0;
      uint32_t mphase = 0;
      auto take_claim = [&]() -> int {
        if constexpr (PAIR) {
          int cl = n_claims;
          if (issuer) {
            if (!mbar_wait_bounded_cluster(&mempty[mslot], mphase ^ 1u, abort_flag, tmo)) {
              ok = false;
              return n_claims;
            }
            cl = atomicAdd(args.work_counter, 1);
            st_cluster_u32(cluster_addr((const void*)&mailbox[mslot], 1), (uint32_t)cl);
            mbar_arrive_cluster(cluster_addr(&mfull[mslot], 1));
          } else {
            if (!mbar_wait_bounded_cluster(&mfull[mslot], mphase, abort_flag, tmo)) {
              ok = false;
              return n_claims;
            }
            cl = mailbox[mslot];
            mbar_arrive_cluster(cluster_addr(&mempty[mslot], 0));
          }
          if (++mslot == UNIT_RING) {
            mslot = 0;
            mphase ^= 1u;
          }
          return cl;
        } else {
          return atomicAdd(args.work_counter, 1);
        }
      };
      int claim = args.dynamic ? take_claim() : worker;
      int u_next = num_units, u_end = num_units;
      auto open_claim = [&]() {
        if (claim < n_claims) {
          u_next = claim < n_pre ? claim : n_pre + (claim - n_pre) * chunk;
          u_end = claim < n_pre ? claim + 1 : min(num_units, u_next + chunk);
        } else {
          u_next = u_end = num_units;
        }
      };
      open_claim();
      int res_key = -1;  // (token tile, problem) whose activation scales are resident in TMEM
      auto wait0 = [&](uint64_t* bar, uint32_t par) -> bool { return mbar_wait_bounded(bar, par, abort_flag, tmo); };
      // the next unit's descriptor is read one unit ahead: its global load lands while this unit's
      // loads are issued
      GemmUnit nxt = {};
      int nxt_pid = 0;
      if (u_next < num_units) nxt = unit_at<BN_MAX, TILE_M>(args, u_next, nxt_pid, prank);
      while (ok) {
        if (!wait0(&uempty[uslot], uphase ^ 1u)) {
          ok = false;
          break;
        }
        const int u = u_next < num_units ? u_next : -1;
        GemmUnit un = nxt;
        const int pid = nxt_pid;
        un.pad1 = pid;
        un.pad2 = u;
        unit_ring[2 * uslot] = make_int4(un.a_row, un.b_row, un.f0, un.nm);
        unit_ring[2 * uslot + 1] = make_int4(un.tile, un.kslice, un.pad1, un.pad2);
        mbar_arrive(&ufull[uslot]);
        if (++uslot == UNIT_RING) {
          uslot = 0;
          uphase ^= 1u;
        }
        if (u < 0) break;
        if (++u_next >= u_end) {
          claim = args.dynamic ? take_claim() : claim + n_workers;
          open_claim();
        }
        if (u_next < num_units) nxt = unit_at<BN_MAX, TILE_M>(args, u_next, nxt_pid, prank);
        const GemmProblem& pr = args.prob[pid];
        const CUtensorMap* mw = pid ? &map_w1 : &map_w0;
        const CUtensorMap* ma = pid ? &map_act1 : &map_act0;
        const uint64_t pol_w = pr.weights_streamed ? pol_first : pol_normal;
        const int nkb = pr.num_k_blocks;
        const int nv = un.nm & 0xFFFF;
        const int nbox = (nv + BOXN - 1) / BOXN;
        // activation scales are loaded unless the previous unit left this tile's resident in TMEM
        bool fill = true;
        if constexpr (FP4 && RES_STAGES > 0) {
          const bool res = pr.sfb_resident != 0 && nkb <= RES_STAGES;
          const int key = (un.tile << 1) | pid;
          fill = !res || key != res_key;
          res_key = res ? key : -1;
        }
        uint32_t bytes = A_STAGE_BYTES + nbox * BOXN * 128 + S::SFA_STAGE_BYTES + (fill ? S::SFB_STAGE_BYTES : 0);
        // pair: one box per CTA, the odd CTA's tokens start half the MMA's N further; the even CTA's
        // stage barrier expects both CTAs' bytes
        int b_row = un.b_row;
        if constexpr (PAIR) {
          b_row += (int)prank * (((nv + 15) & ~15) >> 1);
          bytes = 2u * (A_STAGE_BYTES + BOXN * 128);
        }
        // x coordinate of a stage in the tensor maps: 128 bytes = 64 bf16 elements or 128 FP4 bytes
        const int kx = FP4 ? 128 : BLOCK_K;
        int kb0, kb1;
        unit_k_range(pr, un, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait0(&empty[stage], phase ^ 1u)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * S::STAGE_BYTES;
          uint8_t* sb = sa + A_STAGE_BYTES;
          if constexpr (PAIR) {
            if (issuer) mbar_arrive_expect_tx(&full[stage], bytes);
            const uint32_t bar = cluster_addr(&full[stage], 0);
            tma_load_2d_pair(sa, mw, bar, kb * kx, un.a_row, pol_w);
            tma_load_2d_pair(sb, ma, bar, kb * kx, b_row, pol_a);
          } else {
            mbar_arrive_expect_tx(&full[stage], bytes);
            tma_load_2d(sa, mw, &full[stage], kb * kx, un.a_row, pol_w);
            for (int i = 0; i < nbox; ++i)
              tma_load_2d(sb + i * BOXN * 128, ma, &full[stage], kb * kx, b_row + i * BOXN, pol_a);
          }
          if constexpr (FP4) {
            uint8_t* ssfa = sb + S::B_STAGE_BYTES;
            uint8_t* ssfb = ssfa + S::SFA_STAGE_BYTES;
            bulk_load(ssfa, pr.w_sf + ((long long)(un.a_row >> 7) * pr.w_atoms_k + kb * 4) * (SF_ATOM_BYTES * SF_WREP),
                      S::SFA_STAGE_BYTES, &full[stage]);
            if (fill)
              bulk_load(ssfb, pr.act_sf + ((long long)un.tile * pr.act_sf_stages + kb) * S::SFB_STAGE_BYTES,
                        S::SFB_STAGE_BYTES, &full[stage]);
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) atomicOr(args.status, DEV_STATUS_TIMEOUT);
      if (!ok && issuer) {
        // Give every load still in flight a bounded chance to land before the CTA exits (a pair's
        // loads all complete on the even CTA's barriers).
        volatile int never = 0;
        int s = stage, p = phase;
        for (int i = 0; i < STAGES && i < issued; ++i) {
          if (--s < 0) {
            s = STAGES - 1;
            p ^= 1;
          }
          mbar_wait_bounded(&full[s], p, &never, 100000000ull);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (PAIR && !issuer && lane == 0) {
      // the odd CTA of a pair issues nothing; it only keeps its unit ring moving
      int uslot = 0;
      uint32_t uphase = 0;
      while (true) {
        if (!mbar_wait_bounded(&ufull[uslot], uphase, abort_flag, tmo)) {
          atomicOr(args.status, DEV_STATUS_TIMEOUT);
          break;
        }
        const int u = unit_ring[2 * uslot + 1].w;
        mbar_arrive(&uempty[uslot]);
        if (++uslot == UNIT_RING) {
          uslot = 0;
          uphase ^= 1u;
        }
        if (u < 0) break;
      }
    } else if (lane == 0) {
      int sf_slot = 0;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      int uslot = 0;
      uint32_t uphase = 0;
      int res_key = -1;
      while (ok) {
        if (!mbar_wait_bounded(&ufull[uslot], uphase, abort_flag, tmo)) {
          ok = false;
          break;
        }
        const int4 e0 = unit_ring[2 * uslot], e1 = unit_ring[2 * uslot + 1];
        mbar_arrive(&uempty[uslot]);
        if (++uslot == UNIT_RING) {
          uslot = 0;
          uphase ^= 1u;
        }
        if (e1.w < 0) break;
        const GemmUnit un = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
        const int pid = e1.z;
        const int nkb = args.prob[pid].num_k_blocks;
        const int nv = un.nm & 0xFFFF;
        const uint32_t n_mma = (uint32_t)((nv + 15) & ~15);
        const uint32_t idesc = FP4 ? idesc_nvf4(BLOCK_M, n_mma) : idesc_bf16_f32(TILE_M, n_mma);
        const int nra = (int)((n_mma + 127) >> 7);
        // res: this unit's activation scales live in the resident columns (filled by the tile's first
        // unit, whose copies the tensor pipe runs after the previous tile's MMAs)
        bool res = false, fill = true;
        if constexpr (FP4 && RES_STAGES > 0) {
          res = args.prob[pid].sfb_resident != 0 && nkb <= RES_STAGES;
          const int key = (un.tile << 1) | pid;
          fill = !res || key != res_key;
          res_key = res ? key : -1;
        }
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, tmo)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * S::ACC_COLS);
        int mma_i = 0;  // MMA index within the tile: partial accumulator mma_i % ACC_SPLIT
        int kb0, kb1;
        unit_k_range(args.prob[pid], un, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, tmo)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * S::STAGE_BYTES);
          const uint64_t da = smem_desc_sw128(sa);
          const uint64_t db = smem_desc_sw128(sa + A_STAGE_BYTES);
          if constexpr (FP4) {
            const uint32_t ssfa = sa + A_STAGE_BYTES + S::B_STAGE_BYTES;
            const uint32_t ssfb = ssfa + S::SFA_STAGE_BYTES;
            const uint32_t t_sfa = tmem_base + S::SFA_COL0 + (uint32_t)(sf_slot * 16);
            // activation scales of MMA k of this stage: t_sfb + 4 * k * sfb_pitch
            uint32_t t_sfb;
            int sfb_pitch;
            if (res) {
              t_sfb = tmem_base + S::SFB_COL0 + (uint32_t)(16 * kb * S::NRA);
              sfb_pitch = S::NRA;
            } else {
              t_sfb = tmem_base + S::SFB_COL0 + (uint32_t)(sf_slot * 16 * S::NRA);
              sfb_pitch = S::SFB_REP > 1 ? S::NRA : nra;
            }
            if (++sf_slot == S::SF_SLOTS) sf_slot = 0;
            // weight scales: two copies of two replicated atoms each (K atoms 0-1, then 2-3)
            tcgen05_cp_128x256b(t_sfa, smem_desc_sf_pair(ssfa));
            tcgen05_cp_128x256b(t_sfa + 8, smem_desc_sf_pair(ssfa + 2 * SF_ATOM_BYTES * SF_WREP));
            if constexpr (S::SFB_REP > 1) {
              // both row atoms of K atom k (replicated, 2 KB apart) in one copy: columns 8k .. 8k + 7
#pragma unroll
              for (int k = 0; k < 4; ++k)
                tcgen05_cp_128x256b(t_sfb + 8 * k, smem_desc_sf_pair(ssfb + k * 2 * SF_ATOM_BYTES * SF_WREP));
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                if (fill)
                  for (int ra = 0; ra < nra; ++ra)
                    tcgen05_cp_32x128b_x4(t_sfb + 4 * (k * sfb_pitch + ra),
                                          smem_desc_sf_atom(ssfb + (k * S::NRA + ra) * SF_ATOM_BYTES));
              }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k, ++mma_i)  // K = 64 E2M1 per MMA: +32 bytes = +2 in the address field
              umma_nvf4(d_tmem + (uint32_t)((mma_i % ACC_SPLIT) * BN_MAX), da + 2 * k, db + 2 * k, idesc, t_sfa + 4 * k,
                        t_sfb + 4 * k * sfb_pitch, mma_i >= ACC_SPLIT);
          } else if constexpr (PAIR) {
#pragma unroll
            for (int k = 0; k < BLOCK_K / 16; ++k, ++mma_i)
              umma_bf16_pair(d_tmem, da + 2 * k, db + 2 * k, idesc, mma_i >= 1);
          } else {
#pragma unroll
            for (int k = 0; k < BLOCK_K / 16; ++k, ++mma_i)  // K = 16 bf16 per MMA: +32 bytes = +2 in the address field
              umma_bf16(d_tmem + (uint32_t)((mma_i % ACC_SPLIT) * BN_MAX), da + 2 * k, db + 2 * k, idesc,
                        mma_i >= ACC_SPLIT);
          }
          // the stage is free again in both CTAs of a pair once these MMAs have read it
          if constexpr (PAIR) umma_commit_pair(&empty[stage], 3);
          else umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if constexpr (PAIR) umma_commit_pair(&tfull[acc], 3);
        else umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) atomicOr(args.status, DEV_STATUS_TIMEOUT);
      // every MMA this thread issued completes before TMEM is released
      if constexpr (PAIR) umma_commit_pair(drain, 1);
      else umma_commit(drain);
      volatile int never = 0;
      mbar_wait_bounded(drain, 0, &never, 100000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..)
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int ew = warp - 2;
    const int c_first = ew >> 2, c_step = EPIW >> 2;  // this warp's 32-token chunks of a tile
    uint8_t* stg = smem + S::EPI_OFF + ew * EPI_STAGE_BYTES;
    int acc = 0;
    uint32_t acc_phase = 0;
    int uslot = 0;
    uint32_t uphase = 0;
    while (true) {
      // every wait's outcome is made warp-uniform: the lanes go on to warp-collective TMEM loads
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&ufull[uslot], uphase, abort_flag, tmo))) {
        if (lane == 0) atomicOr(args.status, DEV_STATUS_TIMEOUT);
        break;
      }
      const int4 e0 = unit_ring[2 * uslot], e1 = unit_ring[2 * uslot + 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(&uempty[uslot]);
      if (++uslot == UNIT_RING) {
        uslot = 0;
        uphase ^= 1u;
      }
      if (e1.w < 0) break;
      const GemmUnit un = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
      const int pid = e1.z;
      const GemmProblem& pr = args.prob[pid];
      const int nv = un.nm & 0xFFFF;
      const int mv = un.nm >> 16;
      float oscale = 1.0f;
      if constexpr (FP4) oscale = __ldg(pr.w_gscale + un.a_row / pr.w_rows_per_g) * __ldg(pr.act_gscale);
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, tmo))) {
        if (lane == 0) atomicOr(args.status, DEV_STATUS_TIMEOUT);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * S::ACC_COLS);
      // partial accumulators that received at least one MMA (every tile has >= 4 MMAs)
      int ekb0, ekb1;
      unit_k_range(pr, un, ekb0, ekb1);
      const int n_part = min(ACC_SPLIT, (ekb1 - ekb0) * 4);
      const int nchunks = (nv + 31) >> 5;
      const bool feat_ok = (q * 32) < mv;
      const int f = un.f0 + q * 32;  // first feature of this warp's 32
      if (c_first >= nchunks) {
        // no chunk of this tile for this warp: the accumulator is free as far as it is concerned
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_remote(cluster_addr(&tempty[acc], 0));
          else mbar_arrive(&tempty[acc]);
        }
      }
      for (int c = c_first; c < nchunks; c += c_step) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tbase + (uint32_t)(c * 32), r);
        tmem_ld_wait();
        for (int pp = 1; pp < n_part; ++pp) {
          uint32_t r2[32];
          tmem_ld_32x32b_x32(tbase + (uint32_t)(pp * BN_MAX + c * 32), r2);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) + __uint_as_float(r2[j]));
        }
        if (c + c_step >= nchunks) {
          // accumulator fully read by this warp: hand it back to the MMA issuer
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (PAIR) mbar_arrive_remote(cluster_addr(&tempty[acc], 0));
            else mbar_arrive(&tempty[acc]);
          }
        }
        if constexpr (FP4) {
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * oscale);
        }
        const int row0 = un.b_row + c * 32;
        const int nrows = min(32, nv - c * 32);
        const bool f32_out = pr.epi == EPI_F32;
        if (pr.epi == EPI_ROWSCALE_BF16) {
          const float mys = (lane < nrows) ? pr.row_scale[row0 + lane] : 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * __shfl_sync(0xffffffffu, mys, j));
        } else if (pr.epi == EPI_ADD_BF16) {
          if (feat_ok && q * 32 + lane < mv) {
            // all 32 loads (one coalesced 128-byte row segment each) are in flight before the
            // first add, so the chunk pays one memory latency rather than 32
            const float* ad = pr.addend + (long long)row0 * pr.ld_add + f + lane;
            float av[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) av[j] = __ldg(ad + (long long)(j < nrows ? j : 0) * pr.ld_add);
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) + av[j]);
          }
        } else if (pr.epi == EPI_SQRELU_BF16 || pr.epi == EPI_SQRELU_NVFP4) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float v = fmaxf(__uint_as_float(r[j]), 0.f);
            r[j] = __float_as_uint(v * v);
          }
        }
        __syncwarp();
        if (pr.epi == EPI_SQRELU_NVFP4) {
          // transpose through shared memory (XOR-swizzled columns: conflict-free both ways); lane j then
          // quantises token j's two 16-feature blocks and writes 16 code bytes and 2 scale bytes
          float* s32 = reinterpret_cast<float*>(stg);
#pragma unroll
          for (int j = 0; j < 32; ++j) s32[j * 32 + (lane ^ j)] = __uint_as_float(r[j]);
          __syncwarp();
          if (feat_ok && lane < nrows) {
            uint32_t cw[4];
            uint32_t sbs = 0;
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              float v[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] = s32[lane * 32 + ((b * 16 + i) ^ lane)];
              uint32_t cb[2];
              sbs |= nvfp4_block_fast(v, 1.0f, cb) << (8 * b);
              cw[2 * b] = cb[0];
              cw[2 * b + 1] = cb[1];
            }
            const long long row = row0 + lane;
            *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(pr.out) + row * pr.ldo + f / 2) =
                make_uint4(cw[0], cw[1], cw[2], cw[3]);
            // the two blocks are adjacent bytes of one atom row (f is a multiple of 32)
            for (int rp = 0; rp < S::SFB_REP; ++rp)
              *reinterpret_cast<uint16_t*>(pr.out_sf + act_sf_offset(un.tile, c * 32 + lane, f / 16, pr.out_sf_stages,
                                                                     S::NRA, rp, S::SFB_REP)) = (uint16_t)sbs;
          }
        } else if (f32_out) {
          float* s32 = reinterpret_cast<float*>(stg);
#pragma unroll
          for (int j = 0; j < 32; ++j) s32[j * 32 + lane] = __uint_as_float(r[j]);
          __syncwarp();
          float* dst = reinterpret_cast<float*>(pr.out) + un.kslice * pr.split_stride;
          const long long ld = pr.ldo;
          const int col = pr.out_col0 + f;
          if (feat_ok && q * 32 + (lane & 7) * 4 < mv) {  // this lane's 4 features are valid
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int j = it * 4 + (lane >> 3);
              if (j < nrows) {
                const uint4 v = *reinterpret_cast<const uint4*>(s32 + j * 32 + (lane & 7) * 4);
                *reinterpret_cast<uint4*>(dst + (long long)(row0 + j) * ld + col + (lane & 7) * 4) = v;
              }
            }
          }
        } else {
          uint16_t* s16 = reinterpret_cast<uint16_t*>(stg);
#pragma unroll
          for (int j = 0; j < 32; ++j) s16[j * 32 + lane] = f32_to_bf16_rn(__uint_as_float(r[j]));
          __syncwarp();
          uint16_t* dst = reinterpret_cast<uint16_t*>(pr.out);
          const int col = pr.out_col0 + f;
          if (feat_ok && q * 32 + (lane & 3) * 8 < mv) {  // this lane's 8 features are valid
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              const int j = it * 8 + (lane >> 2);
              if (j < nrows) {
                const uint4 v = *reinterpret_cast<const uint4*>(s16 + j * 32 + (lane & 3) * 8);
                *reinterpret_cast<uint4*>(dst + (long long)(row0 + j) * pr.ldo + col + (lane & 3) * 8) = v;
              }
            }
          }
        }
        __syncwarp();
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  // a pair's MMAs read both CTAs' shared memory and write both CTAs' TMEM: neither CTA releases
  // either before the even CTA's MMAs have drained
  if constexpr (PAIR) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
    else tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
}

}  // namespace lmoe
