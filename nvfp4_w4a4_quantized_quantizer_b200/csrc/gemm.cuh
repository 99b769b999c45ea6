// gemm.cuh -- block-scaled FP4 x FP4 GEMM with the segment epilogue.
//
// y[m, n] = op_s( alpha_s * sum_k e2m1(A[m,k]) sa[m,k/16] e2m1(W[n,k]) sw[n,k/16] )
// for column n in module s.  This is the NVFP4 W4A4 linear layer of the
// paper "Why Gated DeltaNet Survives 4-Bit Quantization" (nefut abstract:
// all linear layers W4A4), with the per-module global-scale repair of fused
// projections (bayesiansapien wiki, "Two practical repairs") and the GDN
// gates (wiki, mechanism study part 2) in the epilogue.
//
// Two kernels:
//   k_gemm_tc<CG> persistent, warp-specialised; one CTA per SM.  CG = 1: a
//                 CTA computes one 128 x 256 output tile at a time; CG = 2: a
//                 cluster of two CTAs computes one 256 x 256 tile with
//                 cta_group::2 MMAs (each CTA loads half of the weight rows).
//                 Producer warps stream the activation and weight codes and
//                 their scale atoms with TMA (128-byte swizzle for the codes)
//                 into a shared-memory ring; four scale-writer warps store
//                 each stage's scale bytes into a per-stage TMEM region
//                 (tcgen05.st) while the MMA warp issues
//                 tcgen05.mma.kind::mxf4nvf4 (K = 64 per instruction) into a
//                 128 x 256 fp32 TMEM accumulator per CTA; eight epilogue
//                 warps drain the accumulator (each lane = one row, 128
//                 columns), release it to the MMA warp, then apply alpha / op
//                 and store.
//   k_gemm_small  M <= 64 (decode shapes): operands swapped so the weight
//                 rows fill the 128-row MMA side and the tokens are the MMA N
//                 dimension (16/32/64); one CTA per 128 weight rows streams
//                 the whole K range through a ring of 7-9 stages.
// Every wait is bounded (mbar_wait); a wait that runs out records the
// device error word, raises the abort flag (of both CTAs of a pair) and the
// kernel returns after draining its own copies and MMAs and freeing TMEM.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "quantize.cuh"

namespace nvfp4 {

constexpr int MAX_SEG = 32;

struct SegTable {
  int nseg;
  int n_off[MAX_SEG + 1];  // n_off[nseg] = N
  float alpha[MAX_SEG];
  int op[MAX_SEG];
  const float* a_log[MAX_SEG];
  const float* dt_bias[MAX_SEG];
};

struct GemmArgs {
  const uint8_t* sfa;  // activation (or, swapped, token) scale atoms
  const uint8_t* sfb;  // weight scale atoms
  int M, N, K;
  void* y;
  int64_t ldy;
  int out_fp32;
  int sector_stores;   // y base 32-byte aligned and rows a multiple of 32 bytes
  int n_fastest;       // tile raster: 0 = M fastest (consecutive CTAs share a weight tile),
                       // 1 = N fastest (they share an activation tile)
  // Stream-K tail (CTA-pair kernel).  With sk_tiles > 0 the last sk_tiles
  // tiles [num_tiles - sk_tiles, num_tiles) are not run whole: their
  // sk_tiles * num_kt k-tiles are cut into `units` contiguous ranges of
  // (nearly) equal length, range u = [sk_len * u / units, sk_len * (u + 1) /
  // units), one per CTA pair, beside the pair's whole data-parallel tiles
  // (dp_tiles = num_tiles - sk_tiles, a multiple of the pair count, walked
  // u, u + units, ...).  sk_tiles >= units, so a range is at least one tile
  // long and a tile is shared by at most two pairs.  The pair whose range
  // starts inside a tile runs those (tail) k-tiles as its very first item
  // and publishes the fp32 partial tile in slot u of the caller's
  // workspace, then raises the slot's flag; the pair whose range ends
  // inside it runs its (head) k-tiles as its very last item, waits for the
  // flag of slot u + 1 (raised long before), adds the partial to its own
  // accumulator (head + tail, the same order whatever the timing) and
  // applies the epilogue.  A short item right after another one would wait
  // for the epilogue of the one before to drain the single accumulator;
  // first and last, the short items overlap whole tiles instead.  The
  // consumer sets the flag back to zero, so the flags are zero between
  // launches.  sk_tiles == 0: every tile whole.
  int sk_tiles;
  float* partial;      // [slot][2 CTAs][2 column halves][32 chunks][128 rows] float4
  unsigned* flags;     // [slot][2 CTAs]
  uint64_t wait_ns;
  // SwiGLU epilogue (k_gemm_tc<2, true>): the weight is [gate; up], H rows
  // each; tile column nb covers h columns [128 nb, 128 nb + 128) -- the even
  // CTA loads those gate rows, the odd CTA the matching up rows -- and the
  // epilogue writes h = bf16(silu(g) * u), g = bf16(alpha_gate * acc_gate),
  // u = bf16(alpha_up * acc_up), quantised under h_gs: codes [M, H/2] and
  // scales in the atom layout (the down projection's activation operand).
  int H;
  float alpha_gate, alpha_up, h_gs;
  uint8_t* h_codes;
  uint8_t* h_scales;
};

// ------------------------------------------------------------- epilogue op
// GDN gates: beta = sigmoid(v); g = -exp(A_log[h]) * softplus(v + dt_bias[h]),
// softplus(z) = max(z, 0) + log(1 + exp(-|z|)).  They use the fast
// exponential, logarithm and division: for the arguments that matter their
// errors change beta by under 1e-6 and g by under ~5e-6 absolute, far below
// what the GEMM's own 1e-3 rms tolerance moves either gate, and each gate is
// then a handful of instructions instead of a few hundred cycles of
// dependent full-precision library code (a column's gates for 64 tokens made
// one CTA of the decode GEMM the last to finish).
__device__ __forceinline__ float gate_sigmoid(float v) {
  return __fdividef(1.0f, 1.0f + __expf(-v));
}

__device__ __forceinline__ float gate_decay(float v, float ea, float dtb) {
  const float z = v + dtb;
  return -ea * (fmaxf(z, 0.0f) + __logf(1.0f + __expf(-fabsf(z))));
}

__device__ __forceinline__ float apply_op(float v, int op, const float* a_log,
                                          const float* dt_bias, int h) {
  if (op == 1) return gate_sigmoid(v);
  if (op == 2) return gate_decay(v, __expf(__ldg(a_log + h)), __ldg(dt_bias + h));
  return v;
}

// Gate epilogue for 16 consecutive columns, kept out of line: only the few
// gate columns take it, and inlining it into the unrolled store loops would
// multiply the kernels' code size.
__device__ __noinline__ void apply_op_16(float* o, int op, const float* a_log,
                                         const float* dt_bias, int h0) {
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i] = apply_op(o[i], op, a_log, dt_bias, h0 + i);
}

// Gate of one column for 16 tokens (op 1 sigmoid, op 2 decay with this
// head's exp(A_log) and dt_bias).  Its one caller runs it in a loop that is
// not unrolled, so it is inlined there.
__device__ __forceinline__ void gate_16(float (&o)[16], int op, float ea, float dtb) {
  if (op == 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = gate_sigmoid(o[i]);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = gate_decay(o[i], ea, dtb);
  }
}

// Advance `seg` so that n lies in [n_off[seg], n_off[seg+1]).
__device__ __forceinline__ int seg_advance(const SegTable& t, int seg, int n) {
  while (seg + 1 < t.nseg && n >= t.n_off[seg + 1]) ++seg;
  return seg;
}

// ============================================================ k_gemm_tc
// Warp roles (16 warps, four warpgroups):
//   WG0  warp 0 producer A: TMA of the activation codes; warp 1 MMA issuer
//        and TMEM owner (the whole warp runs the loop, one elected lane
//        issues each MMA and commit); warp 2 producer B: TMA of the weight
//        codes; warp 3 producer S: TMA of both operands' scale atoms on a
//        barrier of their own, so the scale writers need not wait for the
//        codes.
//   WG1  warps 4-7 scale writers: warp w reads, from the stage in shared
//        memory, the scale bytes TMEM lane quarter w % 4 needs and writes
//        them with tcgen05.st into that stage's TMEM scale region.  A k-tile
//        needs 12 tcgen05.cp copies of scale atoms, each holding the issuing
//        thread ~100-150 cycles (issued by the MMA thread they made the
//        prefill GEMM about twice as slow); register stores of the same
//        bytes take ~40 cycles per stage and run beside the MMAs.
//   WG2-3 warps 8-15 epilogue: warp w drains lane quarter w % 4, column
//        half (w - 8) / 4.
// TMEM: accumulator columns [0, 256); stage s scale region [256 + 48 s, +48):
// 16 columns of activation scales (MMA kk reads column 4 kk + quarter) then
// 32 of weight scales (MMA kk reads columns 8 kk + n / 32).
//
// CG = 1: one CTA computes a 128 x 256 tile.
// CG = 2: a cluster of two CTAs computes a 256 x 256 tile with cta_group::2
// MMAs issued by the even CTA: each CTA loads its own 128 activation rows,
// half of the tile's 256 weight rows and all 256 weight rows' scales.  Per
// k-tile a CTA then brings in 38 KB instead of 54 KB for the same number of
// tensor-core cycles (prefill 4096 x 5120 x 5120: 498 MB of L2 -> shared
// memory traffic instead of 708 MB, 49.6 us instead of 57).  The odd CTA's
// scale writers and epilogue warps arrive on the even CTA's barriers
// through the cluster's shared window; the MMA commits arrive on both CTAs'
// barriers.
//
// Tiles are walked M fastest (consecutive CTAs share a weight tile and the
// activations stay in L2) or, when GemmArgs::n_fastest is set, N fastest
// (they share an activation tile: for activations too large for the L2).
// One item of work of a CTA (pair): k-tiles [kt0, kt1) of one tile, run
// whole (ITEM_WHOLE), as the tail of a stream-K tile whose partial sum is
// published (ITEM_TAIL), or as its head, summed with that partial
// (ITEM_HEAD).  A pair's items in order: the tail of its stream-K range (if
// the range starts inside a tile), its whole data-parallel tiles, the whole
// tiles of its range, the head of its range (if it ends inside a tile).
enum ItemKind : int { ITEM_WHOLE = 0, ITEM_TAIL = 1, ITEM_HEAD = 2 };

struct WorkItem {
  int tile;
  int kt0, kt1;   // k-tiles [kt0, kt1)
  int kind;
};

struct WorkPlan {
  int n_dp;        // whole data-parallel tiles: unit, unit + units, ...
  int sk_base;     // first tile of the stream-K range (absolute index)
  int tail_kt0;    // > 0: the range starts with the tail [tail_kt0, num_kt) of tile sk_base
  int n_whole;     // whole tiles of the range after the tail
  int head_kt1;    // > 0: the range ends with the head [0, head_kt1) of the next tile
  int n_items;
};

__device__ __forceinline__ WorkPlan work_plan(const GemmArgs& g, int unit, int units,
                                              int num_tiles, int num_kt) {
  WorkPlan p;
  if (g.sk_tiles <= 0) {
    p.n_dp = unit < num_tiles ? (num_tiles - 1 - unit) / units + 1 : 0;
    p.sk_base = 0;
    p.tail_kt0 = p.n_whole = p.head_kt1 = 0;
    p.n_items = p.n_dp;
    return p;
  }
  const int dp_tiles = num_tiles - g.sk_tiles;            // a multiple of units
  p.n_dp = dp_tiles / units;
  const int64_t len = static_cast<int64_t>(g.sk_tiles) * num_kt;
  const int s0 = static_cast<int>(len * unit / units);
  const int s1 = static_cast<int>(len * (unit + 1) / units);
  const int a = s0 / num_kt;                               // tile (within the range) of s0
  p.tail_kt0 = s0 - a * num_kt;
  const int first_whole = p.tail_kt0 ? a + 1 : a;
  const int b = s1 / num_kt;                               // tile of the range's end
  p.head_kt1 = s1 - b * num_kt;
  p.n_whole = b - first_whole;
  p.sk_base = dp_tiles + a;
  p.n_items = p.n_dp + (p.tail_kt0 ? 1 : 0) + p.n_whole + (p.head_kt1 ? 1 : 0);
  return p;
}

__device__ __forceinline__ WorkItem work_item(const WorkPlan& p, int unit, int units, int num_kt,
                                              int i) {
  WorkItem w;
  w.kt0 = 0;
  w.kt1 = num_kt;
  w.kind = ITEM_WHOLE;
  if (p.tail_kt0) {
    if (i == 0) {
      w.tile = p.sk_base;
      w.kt0 = p.tail_kt0;
      w.kind = ITEM_TAIL;
      return w;
    }
    --i;
  }
  if (i < p.n_dp) {
    w.tile = unit + i * units;
    return w;
  }
  const int j = i - p.n_dp;
  w.tile = p.sk_base + (p.tail_kt0 ? 1 : 0) + j;
  if (j >= p.n_whole) {
    w.kt1 = p.head_kt1;
    w.kind = ITEM_HEAD;
  }
  return w;
}

// SwiGLU epilogue of one output row: g = bf16(alpha_gate * acc) for the 64
// gate columns in v[0..63], u = bf16(alpha_up * acc) for the up columns in
// v[64..127], h = bf16(silu(g) * u) (silu_mul_f32, as the standalone MLP
// glue kernel computes it), then NVFP4 quantisation of h's four 16-blocks
// under g.h_gs with exactly k_quantize's arithmetic: 32 code bytes at
// h_codes[gm, h0 / 2] and the four scale bytes (one 32-bit word) at the
// atom-layout position of blocks h0/16 .. h0/16 + 3.  Rows gm >= M store
// only their scale word (zero).
__device__ __forceinline__ void swiglu_store_row(const GemmArgs& g, int64_t gm, int h0,
                                                 const uint32_t (&v)[128]) {
  const float c = __fmul_rn(6.0f, g.h_gs);
  uint32_t codes[8];
  uint32_t word = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    float h[16];
    uint32_t amax_bits = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float gv = __bfloat162float(__float2bfloat16_rn(__fmul_rn(g.alpha_gate, __uint_as_float(v[16 * b + i]))));
      const float uv = __bfloat162float(__float2bfloat16_rn(__fmul_rn(g.alpha_up, __uint_as_float(v[64 + 16 * b + i]))));
      h[i] = __bfloat162float(__float2bfloat16_rn(silu_mul_f32(gv, uv)));
      // |h| max on the bit patterns (h is bf16-valued: exact)
      const uint32_t mag = __float_as_uint(h[i]) & 0x7FFFFFFFu;
      amax_bits = mag > amax_bits ? mag : amax_bits;
    }
    const uint32_t sc = cvt_e4m3(__fdiv_rn(__uint_as_float(amax_bits), c));
    const float r = block_reciprocal(sc, g.h_gs);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float f[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) f[k] = __fmul_rn(h[8 * hh + k], r);
      codes[2 * b + hh] = sc == 0 ? 0u : cvt_e2m1x8(f);
    }
    word |= sc << (8 * b);
  }
  if (gm < g.M) {
    uint4* dst = reinterpret_cast<uint4*>(g.h_codes + gm * (g.H / 2) + h0 / 2);
    dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
    dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
  }
  *reinterpret_cast<uint32_t*>(g.h_scales + sf_offset(gm, h0 / 16, g.H)) = word;
}

namespace tc {
constexpr int BM = 128;                 // rows of A per CTA
constexpr int BN = 256;                 // tile columns (MMA N)
constexpr int BK = 256;                 // fp4 elements per stage (128 bytes per row)
constexpr int BKB = BK / 2;
constexpr int SFW_WARP0 = 4;            // scale writers: warps 4-7
constexpr int EPI_WARP0 = 8;            // epilogue: warps 8-15
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 512;
constexpr uint32_t REGS_SMALL = 72;     // WG0 and WG1 after setmaxnreg
constexpr uint32_t REGS_EPI = 184;      // WG2 and WG3 after setmaxnreg
static_assert(2 * 128 * REGS_SMALL + 2 * 128 * REGS_EPI <= 65536, "register split");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;
constexpr uint32_t SF_COL = 256;        // + SF_STRIDE * stage
constexpr int BAR_BYTES = 256;

template <int CG>
struct Cfg {
  static constexpr int B_ROWS = BN / CG;                   // weight rows loaded per CTA
  static constexpr int A_BYTES = BM * BKB;                 // 16 KB
  static constexpr int B_BYTES = B_ROWS * BKB;             // 32 / 16 KB
  static constexpr int SFA_BYTES = 4 * 512;                // 4 atoms (K = 64 each) x 128 rows
  // Weight scales: both 128-row blocks of the tile's 256 weight rows, in
  // either kernel.  In a CTA pair each CTA's half of a cta_group::2 MMA (its
  // own 128 output rows) reads the scales of all 256 weight rows from its
  // own TMEM: a layout experiment that left one half of them out (NaN scale
  // codes) in either CTA turned half of that CTA's output columns into NaN.
  static constexpr int SFB_BYTES = 2 * 4 * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;  // 54 / 38 KB
  static constexpr int STAGES = CG == 1 ? 4 : 5;
  // TMEM scale region per stage: SFA 16 columns (4 per MMA), then SFB 32
  // columns (8 per MMA: 4 per 128-row block)
  static constexpr uint32_t SFB_PER_MMA = 8;
  static constexpr uint32_t SF_STRIDE = 16 + 4 * SFB_PER_MMA;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");
  static_assert(SF_COL + STAGES * SF_STRIDE <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};
}  // namespace tc

// tmA / tmB: code matrices [rows, K/2] (box 128 bytes x 128 / (256 / CG)
// rows, 128-byte swizzle).  tmSA / tmSB: scale buffers viewed as [row blocks]
// [K/64 atoms][64 u64] (box 64 x 4 x 1 / 2, i.e. one stage's atoms of 1 / 2
// row blocks).  CG = 2 must be launched with clusters of 2 CTAs.  SWIGLU
// (CG = 2 only): the epilogue is the SwiGLU one described at GemmArgs::H.
template <int CG, bool SWIGLU = false>
__global__ void __launch_bounds__(tc::THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
              const GemmArgs g, const __grid_constant__ SegTable seg) {
  static_assert(!SWIGLU || CG == 2, "the SwiGLU epilogue pairs gate and up rows across a CTA pair");
  using namespace tc;
  using C = Cfg<CG>;
  constexpr int STAGES = C::STAGES;
  constexpr int STAGE_BYTES = C::STAGE_BYTES;
  constexpr int A_BYTES = C::A_BYTES;
  constexpr int B_BYTES = C::B_BYTES;
  constexpr int SFA_BYTES = C::SFA_BYTES;
  constexpr int SFB_BYTES = C::SFB_BYTES;
  constexpr uint32_t SF_STRIDE = C::SF_STRIDE;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  // bars: full[S], empty[S], sf_ready[S], sf_full[S], tmem_full, tmem_empty, drain_mma
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * STAGES + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = CG == 1 ? 0u : cluster_ctarank();
  const int unit = static_cast<int>(blockIdx.x) / CG;     // CTA (pair) index
  const int units = static_cast<int>(gridDim.x) / CG;
  const int num_m = (g.M + BM * CG - 1) / (BM * CG);
  const int num_n = SWIGLU ? g.H / 128 : (g.N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kt = (g.K + BK - 1) / BK;
  const WorkPlan plan = work_plan(g, unit, units, num_tiles, num_kt);
  const int n_items = plan.n_items;

  auto full_bar = [&](int s) { return smem_addr(bars + s); };
  auto empty_bar = [&](int s) { return smem_addr(bars + STAGES + s); };
  auto sf_bar = [&](int s) { return smem_addr(bars + 2 * STAGES + s); };
  auto sfull_bar = [&](int s) { return smem_addr(bars + 3 * STAGES + s); };
  const uint32_t tmem_full = smem_addr(bars + 4 * STAGES);
  const uint32_t tmem_empty = smem_addr(bars + 4 * STAGES + 1);
  const uint32_t drain_mma = smem_addr(bars + 4 * STAGES + 2);

  // Barriers that the MMA issuer waits on live in the even CTA; the odd CTA
  // arrives on them through the cluster window.
  auto arrive_leader = [&](uint32_t bar) {
    if constexpr (CG == 1)
      mbar_arrive(bar);
    else
      mbar_arrive_remote(mapa_shared(bar, 0));
  };
  auto wait_pair = [&](uint32_t bar, uint32_t parity) {
    return mbar_wait_warp(bar, parity, g.wait_ns, abort_flag);
  };
  // A role that gives up raises the abort flag of both CTAs of the pair.
  auto raise_abort = [&](uint32_t site, uint32_t role) {
    if (!*abort_flag) record_error(site, role);
    *abort_flag = 1;
    if constexpr (CG == 2)
      st_shared_remote_u32(mapa_shared(smem_addr(const_cast<int*>(abort_flag)), rank ^ 1u), 1u);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 2);            // both producers arrive (with their bytes)
      mbar_init(empty_bar(s), 1);
      mbar_init(sf_bar(s), 4 * CG);         // the scale writers of every CTA of the pair
      mbar_init(sfull_bar(s), 1);           // the scale producer
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, EPI_WARPS * CG);
    mbar_init(drain_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmSA);
    prefetch_tensormap(&tmSB);
  }
  if (warp == 1) {
    tmem_alloc_cg<CG>(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish_cg<CG>();
  }
  tc_fence_before();
  if constexpr (CG == 1)
    __syncthreads();
  else
    cluster_sync();   // the other CTA's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // With launch overlap the next kernel may now be scheduled as SMs free up.
  // Only the weight codes stream before the kernel ahead has finished: the
  // activation and scale producers and the epilogue wait for it
  // (griddep_wait) before they read its outputs or write y, h or the
  // stream-K workspace.
  griddep_launch_dependents();

  // Each warpgroup resizes its registers at the top of its own branch.
  if (warp < SFW_WARP0) regs_dealloc<REGS_SMALL>();
  if (warp == 0 || warp == 2 || warp == 3) {
    // ---------------------------------------------------- TMA producers
    // warp-wide loop; one elected lane issues each copy
    if (warp != 2) griddep_wait();   // activation codes and both operands' scales
    {
      // L2 policy per operand.  With the N-fastest raster (activations too
      // large for L2, e.g. the MLP down projection's 143 MB of codes) each
      // activation tile is read by consecutive pairs at about the same time
      // and then not again: it is marked evict-first, and the weights, re-read
      // for every activation tile, evict-last (down projection 621 vs 639 us).
      // With the M-fastest raster both stay evict-last: marking the weight
      // tiles evict-first made the GDN in-projection 3% slower.
      const uint64_t keep = policy_evict_last();
      const uint64_t pol_a = g.n_fastest ? policy_evict_first() : keep;
      const uint64_t pol_b = keep;
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int it = 0; it < n_items && ok; ++it) {
        const WorkItem w = work_item(plan, unit, units, num_kt, it);
        const int tile = w.tile;
        const int mb = g.n_fastest ? tile / num_n : tile % num_m;
        const int nb = g.n_fastest ? tile % num_n : tile / num_m;
        const int arow = (mb * CG + static_cast<int>(rank)) * BM;
        // SwiGLU: the even CTA's half of the tile is gate rows, the odd CTA's the up rows
        const int brow = SWIGLU ? nb * 128 + (rank ? g.H : 0)
                                : nb * BN + static_cast<int>(rank) * C::B_ROWS;
        for (int kt = w.kt0; kt < w.kt1; ++kt) {
          if (!wait_pair(empty_bar(stage), phase ^ 1u)) {
            raise_abort(SITE_PRODUCER_EMPTY, warp);
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * STAGE_BYTES;
          if (warp == 0) {
            mbar_arrive_expect_tx_warp(full_bar(stage), A_BYTES);
            tma_load_2d_warp(smem_addr(st), &tmA, kt * BKB, arow, full_bar(stage), pol_a);
          } else if (warp == 2) {
            mbar_arrive_expect_tx_warp(full_bar(stage), B_BYTES);
            tma_load_2d_warp(smem_addr(st + A_BYTES), &tmB, kt * BKB, brow, full_bar(stage), pol_b);
          } else {
            // both boxes always transfer their full size (out-of-range atoms read as 0)
            mbar_arrive_expect_tx_warp(sfull_bar(stage), SFA_BYTES + SFB_BYTES);
            tma_load_3d_warp(smem_addr(st + A_BYTES + B_BYTES), &tmSA, 0, kt * 4,
                        mb * CG + static_cast<int>(rank), sfull_bar(stage), pol_a);
            if constexpr (SWIGLU) {
              // the gate rows' scale block, then the up rows' (1-block boxes)
              tma_load_3d_warp(smem_addr(st + A_BYTES + B_BYTES + SFA_BYTES), &tmSB, 0, kt * 4, nb,
                               sfull_bar(stage), pol_b);
              tma_load_3d_warp(smem_addr(st + A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES / 2), &tmSB, 0,
                               kt * 4, g.H / 128 + nb, sfull_bar(stage), pol_b);
            } else {
              // both row blocks of the tile (2-block boxes)
              tma_load_3d_warp(smem_addr(st + A_BYTES + B_BYTES + SFA_BYTES), &tmSB, 0, kt * 4,
                               nb * 2, sfull_bar(stage), pol_b);
            }
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every copy this warp issued must land before the CTA may exit
      const uint32_t mine = (warp == 3) ? 1u : 0u;
      for (int s = 0; s < STAGES && s < issued; ++s) {
        const int64_t uses = (issued - 1 - s) / STAGES + 1;
        const uint32_t bar = mine ? sfull_bar(s) : full_bar(s);
        if (!mbar_wait(bar, static_cast<uint32_t>((uses - 1) & 1), g.wait_ns, nullptr))
          record_error(SITE_DRAIN, warp);
      }
    }
    __syncwarp();
  } else if (warp >= SFW_WARP0 && warp < EPI_WARP0) {
    // ---------------------------------------------------- scale writers
    regs_dealloc<REGS_SMALL>();
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    int stage = 0;
    uint32_t phase = 0;
    for (int it = 0; it < n_items; ++it) {
      const WorkItem w = work_item(plan, unit, units, num_kt, it);
      bool ok = true;
      for (int kt = w.kt0; kt < w.kt1; ++kt) {
        if (!mbar_wait_warp(sfull_bar(stage), phase, g.wait_ns, abort_flag)) {
          raise_abort(SITE_MMA_FULL, warp);
          ok = false;
          break;
        }
        const uint32_t sfa_s = smem_addr(smem + stage * STAGE_BYTES + A_BYTES + B_BYTES);
        const uint32_t sfb_s = sfa_s + SFA_BYTES;
        uint32_t r[48];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // activation row 32 q + lane, MMA kk: 4 scale bytes at atom kk
          const uint32_t a = ld_shared_u32(sfa_s + kk * 512 + lane * 16 + q * 4);
          r[4 * kk + 0] = a;
          r[4 * kk + 1] = a;
          r[4 * kk + 2] = a;
          r[4 * kk + 3] = a;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            // weight rows 128 j + 32 c + lane of the stage's blocks, c = 0..3
            // -> columns SFB_PER_MMA kk + 4 j + c
            const uint4 b = ld_shared_v4(sfb_s + j * 2048 + kk * 512 + lane * 16);
            r[16 + C::SFB_PER_MMA * kk + 4 * j + 0] = b.x;
            r[16 + C::SFB_PER_MMA * kk + 4 * j + 1] = b.y;
            r[16 + C::SFB_PER_MMA * kk + 4 * j + 2] = b.z;
            r[16 + C::SFB_PER_MMA * kk + 4 * j + 3] = b.w;
          }
        }
        const uint32_t col = tmem_base + lane_off + SF_COL + SF_STRIDE * stage;
        tmem_st_x32(col, r);
        tmem_st_x16(col + 32, r + 32);
        tmem_wait_st();
        tc_fence_before();
        // the MMA warp waits on this barrier alone: arrive only once the
        // stage's codes have landed too
        if (!mbar_wait_warp(full_bar(stage), phase, g.wait_ns, abort_flag)) {
          raise_abort(SITE_MMA_FULL, warp);
          ok = false;
          break;
        }
        __syncwarp();
        if (lane == 0) arrive_leader(sf_bar(stage));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    // The tensor pipe accepts about one MMA ahead of the issuing thread, so
    // the issuer's own bookkeeping shows up as pipe idle time: the whole warp
    // runs the loop (warp-uniform descriptors, one elected lane issues each
    // MMA and commit), waits on a single barrier per stage (the scale writers
    // arrive only once both the codes and the scales of the stage are in
    // place), and releases the previous stage right after MMA 0.
    if (rank == 0) {
      const uint32_t idesc = idesc_mxf4nvf4(BM * CG, BN);
      // the start-address field holds (address >> 4) and every stage lies below
      // 256 KB, so a stage's descriptor is the first one plus stage * STAGE_BYTES / 16
      const uint64_t adesc0 = desc_kmajor_sw128(smem_addr(smem));
      const uint64_t bdesc0 = desc_kmajor_sw128(smem_addr(smem + A_BYTES));
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int it = 0; it < n_items && ok; ++it, ++local) {
        const WorkItem w = work_item(plan, unit, units, num_kt, it);
        if (!wait_pair(tmem_empty, static_cast<uint32_t>((local & 1) ^ 1))) {
          raise_abort(SITE_MMA_TMEM_EMPTY, 1);
          break;
        }
        tc_fence_after();
        int prev = -1;
        for (int kt = w.kt0; kt < w.kt1; ++kt) {
          if (!wait_pair(sf_bar(stage), phase)) {
            raise_abort(SITE_MMA_FULL, 1);
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk = min(4, (g.K - kt * BK) / 64);
          const uint64_t soff = static_cast<uint64_t>(stage) * (STAGE_BYTES >> 4);
          const uint64_t ad = adesc0 + soff, bd = bdesc0 + soff;
          const uint32_t col = tmem_base + SF_COL + SF_STRIDE * stage;
          // K = 64 fp4 = 32 bytes per MMA: advance the start address inside the swizzle atom
          mma_mxf4nvf4_warp<CG>(tmem_base + ACC_COL, ad, bd, idesc, col, col + 16, kt != w.kt0);
          if (prev >= 0) tc_commit_all_warp<CG>(empty_bar(prev));
          for (int kk = 1; kk < nk; ++kk)
            mma_mxf4nvf4_warp<CG>(tmem_base + ACC_COL, ad + 2 * kk, bd + 2 * kk, idesc,
                                col + 4 * kk, col + 16 + C::SFB_PER_MMA * kk, 1u);
          prev = stage;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (prev >= 0) tc_commit_all_warp<CG>(empty_bar(prev));
        if (!ok) break;
        tc_commit_all_warp<CG>(tmem_full);
      }
      // all issued tensor-core work must finish before TMEM is freed
      tc_commit_local_warp<CG>(drain_mma);
      if (!mbar_wait(drain_mma, 0, g.wait_ns, nullptr)) record_error(SITE_DRAIN, 1);
    }
    __syncwarp();
  } else if (warp >= EPI_WARP0) {
    // ---------------------------------------------------------- epilogue
    regs_alloc<REGS_EPI>();
    griddep_wait();   // y (or h) and the workspace may still be in use by the kernel ahead
    const int q = warp & 3;                       // TMEM lane quarter this warp may access
    const int half = (warp - EPI_WARP0) >> 2;     // columns [128*half, 128*half + 128)
    const int row_in_tile = q * 32 + lane;
    // The output of one tile row: alpha / op, bf16 RNE (or fp32), store.
    // fetch(grp, a) yields the fp32 accumulator bits of columns
    // 16 grp .. 16 grp + 15 of this thread's 128.
    // Rows past M skip only the stores: fetch may issue warp-collective
    // TMEM loads, so every lane of the warp runs it.
    // With the N-fastest raster the output is marked evict-first too, so it
    // does not push the kept weights out of L2.
    const uint64_t out_pol = g.n_fastest ? policy_evict_first() : policy_evict_normal();
    auto store_row = [&](int mb, int nb, auto&& fetch) {
      const int64_t gm = static_cast<int64_t>(mb * CG + static_cast<int>(rank)) * BM + row_in_tile;
      const bool row_live = gm < g.M;
      const int n0 = nb * BN + half * 128;
      int s = seg_advance(seg, 0, n0);
#pragma unroll
      for (int grp = 0; grp < 8; ++grp) {
        const int n = n0 + grp * 16;
        if (n < g.N) {
          s = seg_advance(seg, s, n);
          const float alpha = seg.alpha[s];
          const int op = seg.op[s];
          const int h0 = n - seg.n_off[s];
          uint32_t a[16];
          fetch(grp, a);
          float o[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __fmul_rn(alpha, __uint_as_float(a[i]));
          if (op != 0) {
            float t[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) t[i] = o[i];
            apply_op_16(t, op, seg.a_log[s], seg.dt_bias[s], h0);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = t[i];
          }
          if (row_live && g.out_fp32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(g.y) + gm * g.ldy + n);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          } else if (row_live) {
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const __nv_bfloat162 p = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
              w[i] = *reinterpret_cast<const uint32_t*>(&p);
            }
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(g.y) + gm * g.ldy + n;
            if (g.sector_stores) {
              st_global_v8_hint(dst, w, out_pol);   // the row's 16 columns = one full 32-byte sector
            } else {
              reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
              reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
          }
        }
      }
    };
    // Stream-K partial tiles: chunk c (columns 4c..4c+3 of this thread's
    // 128) of slot u; for one chunk a warp's 32 rows are 512 contiguous bytes
    auto part_chunk = [&](int u, int c) {
      return reinterpret_cast<float4*>(g.partial) +
             ((((static_cast<size_t>(u) * 2 + rank) * 2 + half) * 32 + c) * BM + row_in_tile);
    };
    int local = 0;
    bool dead = false;   // a wait ran out: skip the work, keep every barrier
    for (int it = 0; it < n_items; ++it, ++local) {
      const WorkItem wi = work_item(plan, unit, units, num_kt, it);
      const int mb = g.n_fastest ? wi.tile / num_n : wi.tile % num_m;
      const int nb = g.n_fastest ? wi.tile % num_n : wi.tile / num_m;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ACC_COL + half * 128;
      bool ok = !dead;
      // The head k-tiles of a stream-K tile (always the pair's last item):
      // the tail partial was published by the next pair as its first item.
      // Wait for its flag and start loading it while this pair's own
      // k-tiles finish; once the accumulator is complete, add the
      // partial to it in TMEM (head + tail), 16 columns at a time with two
      // column groups of it in registers, then run the whole-tile epilogue.
      const bool head = !SWIGLU && wi.kind == ITEM_HEAD;
      const unsigned* flag = g.flags + (unit + 1) * 2 + rank;
      float4 pr[2][4];
      if (head) {
        if (ok && !flag_wait_warp(flag, g.wait_ns, abort_flag)) {
          raise_abort(SITE_SK_FLAG, warp);
          dead = true;
          ok = false;
        }
        if (ok) {
#pragma unroll
          for (int gg = 0; gg < 2; ++gg)
#pragma unroll
            for (int c = 0; c < 4; ++c) pr[gg][c] = __ldcg(part_chunk(unit + 1, gg * 4 + c));
        }
      }
      if (ok && !wait_pair(tmem_full, static_cast<uint32_t>(local & 1))) {
        raise_abort(SITE_EPI_TMEM_FULL, warp);
        dead = true;
        ok = false;
      }
      uint32_t v[128];
      if (ok) {
        tc_fence_after();
        if (head) {
#pragma unroll
          for (int grp = 0; grp < 8; ++grp) {
            uint32_t t[16];
            tmem_ld_x16(taddr + grp * 16, t);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float4 x = pr[grp & 1][c];
              t[4 * c + 0] = __float_as_uint(__uint_as_float(t[4 * c + 0]) + x.x);
              t[4 * c + 1] = __float_as_uint(__uint_as_float(t[4 * c + 1]) + x.y);
              t[4 * c + 2] = __float_as_uint(__uint_as_float(t[4 * c + 2]) + x.z);
              t[4 * c + 3] = __float_as_uint(__uint_as_float(t[4 * c + 3]) + x.w);
            }
            if (grp < 6) {
#pragma unroll
              for (int c = 0; c < 4; ++c)
                pr[grp & 1][c] = __ldcg(part_chunk(unit + 1, (grp + 2) * 4 + c));
            }
            tmem_st_x16(taddr + grp * 16, t);
          }
          tmem_wait_st();
        }
        if constexpr (SWIGLU) {
          // this warp's 64 h columns: gate accumulator columns [64 half, +64)
          // into v[0..63], the matching up columns [128 + 64 half, +64) into v[64..127]
          const uint32_t lane_base = taddr - half * 128;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            tmem_ld_x32(lane_base + half * 64 + c * 32, v + c * 32);
            tmem_ld_x32(lane_base + 128 + half * 64 + c * 32, v + 64 + c * 32);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld_x32(taddr + c * 32, v + c * 32);
        }
        tmem_wait_ld();
        // the accumulator is in registers: the MMA warp may start the next item
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_leader(tmem_empty);
      }
      if constexpr (SWIGLU) {
        // whole tiles only (the host never gives this launch a stream-K
        // range); rows past M inside the last 128-row block still write
        // their (zero) scale bytes: the scale buffer's padding rows must
        // hold zeros
        const int64_t gm = static_cast<int64_t>(mb * CG + static_cast<int>(rank)) * BM + row_in_tile;
        const int64_t rows_padded = (static_cast<int64_t>(g.M) + 127) / 128 * 128;
        if (ok && gm < rows_padded) swiglu_store_row(g, gm, nb * 128 + half * 64, v);
        continue;
      } else if (wi.kind != ITEM_TAIL) {
        if (ok)
          store_row(mb, nb, [&](int grp, uint32_t (&a)[16]) {
#pragma unroll
            for (int i = 0; i < 16; ++i) a[i] = v[grp * 16 + i];
          });
        if (head) {
          // every epilogue warp has read the partial: the flag returns to zero
          asm volatile("bar.sync 1, 256;" ::: "memory");
          if (ok && warp == EPI_WARP0 && lane == 0) st_relaxed_gpu_u32(const_cast<unsigned*>(flag), 0u);
        }
        continue;
      }
      // the tail k-tiles of a stream-K tile (the pair's first item): publish
      // the partial in slot `unit`, then raise its flag
      if (ok) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          __stcg(part_chunk(unit, c),
                 make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]),
                             __uint_as_float(v[4 * c + 2]), __uint_as_float(v[4 * c + 3])));
        __threadfence();
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (ok && !*abort_flag && warp == EPI_WARP0 && lane == 0)
        red_release_gpu_add_u32(g.flags + unit * 2 + rank, 1u);
    }
  }

  // No CTA of a pair leaves (or frees TMEM) while the pair's MMAs, copies or
  // remote arrivals may still touch it.
  tc_fence_before();
  if constexpr (CG == 1)
    __syncthreads();
  else
    cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_cg<CG>(tmem_base, TMEM_COLS);
}

// ========================================================== k_gemm_small
// Warp roles (12 warps): 0 producer W (weight codes + scale atoms), 1 MMA
// issuer, 2 producer X (token codes + scale atoms), 3 idle, 4-7 scale
// writers (tcgen05.st of the stage's scale bytes for lane quarter w % 4),
// 8-11 epilogue (warp w reads TMEM lane quarter w % 4).  TMEM: accumulator
// columns [0, NT); stage s scale region [64 + 32 s, 64 + 32 s + 32): 16
// columns of weight scales (MMA kk reads 4 kk + quarter) then 16 of token
// scales (MMA kk reads 16 + 4 kk + token / 32).
namespace sm {
constexpr int BW = 128;                 // weight rows per CTA (MMA M)
constexpr int DIRECT_M = 8;             // up to this many tokens the epilogue stores directly
constexpr int BK = 256;
constexpr int BKB = BK / 2;
constexpr int W_BYTES = BW * BKB;       // 16 KB
constexpr int SFW_BYTES = 4 * 512;
constexpr int SFX_BYTES = 4 * 512;
constexpr int SFW_WARP0 = 4;
constexpr int EPI_WARP0 = 8;
constexpr int EPI_WARPS = 4;
constexpr int THREADS = 32 * (EPI_WARP0 + EPI_WARPS);
constexpr uint32_t ACC_COL = 0;         // NT columns
constexpr uint32_t SF_COL = 64;         // + 32 * stage
constexpr uint32_t SF_STRIDE = 32;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_PER_SM = 233472;     // 228 KB
constexpr int SMEM_RESERVED = 1024;     // per CTA
// One CTA per SM with the deepest ring that fits: 9 / 8 / 7 stages of 22 /
// 24 / 28 KB for 16 / 32 / 64 tokens.  Each CTA streams one 128-row weight
// block, and its rate is bounded by the bytes it has in flight, so depth
// beats a second CTA per SM: at 16 tokens two CTAs of 5 stages (the next
// call's CTAs streaming beside this call's under launch overlap) took 10.8
// us per call on 16480 x 5120 weights, one of 9 stages 10.2 us, and a
// 10th stage or an L2 run-ahead prefetch of 5-10 k-tiles beyond the ring
// gained nothing or lost (interleaved runs).
template <int NT>
struct Cfg {
  static constexpr int X_BYTES = NT * BKB;   // NT rows x 128 bytes
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES + SFW_BYTES + SFX_BYTES;
  static constexpr int STAGES = NT <= 16 ? 9 : (NT <= 32 ? 8 : 7);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = SF_COL + STAGES * SF_STRIDE <= 256 ? 256u : 512u;
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");
  static_assert(SF_COL + STAGES * SF_STRIDE <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES + SMEM_RESERVED <= SMEM_PER_SM, "shared memory");
  static_assert(NT * BW * 4 <= STAGES * STAGE_BYTES, "the epilogue's transpose fits the ring");
};
}  // namespace sm

// tmW: weight codes [N, K/2]; tmX: token codes [M, K/2].  D (TMEM) is
// [128 weight rows] x [NT tokens]; y[token, n] is written transposed back.
template <int NT>
__global__ void __launch_bounds__(sm::THREADS, 1)
    k_gemm_small(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                 const GemmArgs g, const __grid_constant__ SegTable seg) {
  using namespace sm;
  using C = Cfg<NT>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
  // bars: full[S], empty[S], sf_ready[S], acc_full, drain_mma
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * STAGES + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wt = blockIdx.x;              // weight tile: rows [128 wt, 128 wt + 128)
  const int num_kt = (g.K + BK - 1) / BK;
  const int64_t kb4 = g.K / 64;

  auto full_bar = [&](int s) { return smem_addr(bars + s); };
  auto empty_bar = [&](int s) { return smem_addr(bars + STAGES + s); };
  auto sf_bar = [&](int s) { return smem_addr(bars + 2 * STAGES + s); };
  const uint32_t acc_full = smem_addr(bars + 3 * STAGES);
  const uint32_t drain_mma = smem_addr(bars + 3 * STAGES + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 2);
      mbar_init(empty_bar(s), 1);
      mbar_init(sf_bar(s), 4);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // With launch overlap the next kernel may now be scheduled beside this one.
  // Only the weight stream starts before the kernel ahead has finished: the
  // token producer and the epilogue wait for it (griddep_wait) before they
  // read the token operands or write y.
  griddep_launch_dependents();

  if (warp == 0 || warp == 2) {
    // warp-wide loop; one elected lane issues each copy
    {
      const bool is_w = (warp == 0);
      if (!is_w) griddep_wait();   // the token operands may come from the kernel ahead
      // weights stream through once; tokens are re-read by every CTA
      const uint64_t pol = is_w ? policy_evict_first() : policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      for (int kt = 0; kt < num_kt; ++kt) {
        if (!mbar_wait_warp(empty_bar(stage), phase ^ 1u, g.wait_ns, abort_flag)) {
          if (!*abort_flag) record_error(SITE_PRODUCER_EMPTY, warp);
          *abort_flag = 1;
          break;
        }
        const int nk = min(4, (g.K - kt * BK) / 64);
        uint8_t* st = smem + stage * C::STAGE_BYTES;
        if (is_w) {
          mbar_arrive_expect_tx_warp(full_bar(stage), W_BYTES + nk * 512);
          tma_load_2d_warp(smem_addr(st), &tmW, kt * BKB, wt * BW, full_bar(stage), pol);
          bulk_load_warp(smem_addr(st + W_BYTES + C::X_BYTES), g.sfb + (wt * kb4 + kt * 4) * 512,
                    nk * 512, full_bar(stage), pol);
        } else {
          mbar_arrive_expect_tx_warp(full_bar(stage), C::X_BYTES + nk * 512);
          tma_load_2d_warp(smem_addr(st + W_BYTES), &tmX, kt * BKB, 0, full_bar(stage), pol);
          bulk_load_warp(smem_addr(st + W_BYTES + C::X_BYTES + SFW_BYTES), g.sfa + (kt * 4) * 512,
                    nk * 512, full_bar(stage), pol);
        }
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      for (int s = 0; s < STAGES && s < issued; ++s) {
        const int64_t uses = (issued - 1 - s) / STAGES + 1;
        if (!mbar_wait(full_bar(s), static_cast<uint32_t>((uses - 1) & 1), g.wait_ns, nullptr))
          record_error(SITE_DRAIN, warp);
      }
    }
    __syncwarp();
  } else if (warp >= SFW_WARP0 && warp < EPI_WARP0) {
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    int stage = 0;
    uint32_t phase = 0;
    for (int kt = 0; kt < num_kt; ++kt) {
      if (!mbar_wait_warp(full_bar(stage), phase, g.wait_ns, abort_flag)) {
        if (!*abort_flag) record_error(SITE_MMA_FULL, warp);
        *abort_flag = 1;
        break;
      }
      const uint32_t sfw_s = smem_addr(smem + stage * C::STAGE_BYTES + W_BYTES + C::X_BYTES);
      const uint32_t sfx_s = sfw_s + SFW_BYTES;
      uint32_t r[32];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t a = ld_shared_u32(sfw_s + kk * 512 + lane * 16 + q * 4);
        r[4 * kk + 0] = a;
        r[4 * kk + 1] = a;
        r[4 * kk + 2] = a;
        r[4 * kk + 3] = a;
        const uint4 b = ld_shared_v4(sfx_s + kk * 512 + lane * 16);
        r[16 + 4 * kk + 0] = b.x;
        r[16 + 4 * kk + 1] = b.y;
        r[16 + 4 * kk + 2] = b.z;
        r[16 + 4 * kk + 3] = b.w;
      }
      tmem_st_x32(tmem_base + lane_off + SF_COL + SF_STRIDE * stage, r);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sf_bar(stage));
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  } else if (warp == 1) {
    // the whole warp runs the issuing loop (warp-uniform operands); one
    // elected lane issues each MMA and commit
    {
      const uint32_t idesc = idesc_mxf4nvf4(BW, NT);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kt = 0; kt < num_kt; ++kt) {
        if (!mbar_wait_warp(sf_bar(stage), phase, g.wait_ns, abort_flag) ||
            !mbar_wait_warp(full_bar(stage), phase, g.wait_ns, abort_flag)) {
          if (!*abort_flag) record_error(SITE_MMA_FULL, 1);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const int nk = min(4, (g.K - kt * BK) / 64);
        const uint8_t* st = smem + stage * C::STAGE_BYTES;
        const uint64_t wdesc = desc_kmajor_sw128(smem_addr(st));
        const uint64_t xdesc = desc_kmajor_sw128(smem_addr(st + W_BYTES));
        const uint32_t col = tmem_base + SF_COL + SF_STRIDE * stage;
        for (int kk = 0; kk < nk; ++kk)
          mma_mxf4nvf4_warp<1>(tmem_base + ACC_COL, wdesc + 2 * kk, xdesc + 2 * kk, idesc,
                               col + 4 * kk, col + 16 + 4 * kk, (kt | kk) != 0);
        tc_commit_all_warp<1>(empty_bar(stage));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) tc_commit_all_warp<1>(acc_full);
      tc_commit_all_warp<1>(drain_mma);
      if (!mbar_wait(drain_mma, 0, g.wait_ns, nullptr)) record_error(SITE_DRAIN, 1);
    }
    __syncwarp();
  } else if (warp >= EPI_WARP0) {
    const int q = warp & 3;
    const int r = q * 32 + lane;                 // accumulator row = output column n0 + r
    const int n = wt * BW + r;
    // Thread r holds column n for all NT tokens.  With more than DIRECT_M
    // tokens the tile goes through shared memory (the stage ring is free once
    // every MMA has completed) so that each token's 128 columns leave as
    // 16-byte stores of one contiguous segment instead of M strided 2-byte
    // stores per thread.
    // This column's module, alpha and gate parameters, looked up while the
    // weights stream (each lookup is a dependent constant-bank or global
    // load; after the accumulator is ready they would delay the stores).
    // Columns past N (the last tile's padding) are never stored; they take
    // no gate, so no gate parameter past the module's heads is read.
    const bool live = n < g.N;
    const int s = seg_advance(seg, 0, live ? n : g.N - 1);
    const float alpha = seg.alpha[s];
    const int op = live ? seg.op[s] : 0;     // columns past N take no gate
    const int h = n - seg.n_off[s];
    griddep_wait();   // y may still be read or written by the kernel ahead
    const float ea = op == 2 ? __expf(__ldg(seg.a_log[s] + h)) : 0.0f;
    const float dtb = op == 2 ? __ldg(seg.dt_bias[s] + h) : 0.0f;
    const bool ok = mbar_wait_warp(acc_full, 0, g.wait_ns, abort_flag);
    if (ok) {
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ACC_COL;
      float* t32 = reinterpret_cast<float*>(smem);
      __nv_bfloat16* t16 = reinterpret_cast<__nv_bfloat16*>(smem);
      // Tokens go 16 at a time through a loop that is not unrolled.  This
      // code runs once per CTA, so every instruction of it is fetched cold:
      // unrolled over 64 tokens and three gate kinds it took 2.4 us per CTA
      // (and 8 us in a CTA holding gate columns) against 0.1 us of work.
      // Padding tokens of the last chunk are computed but never stored.
      const int nchunks = ((g.M < NT ? g.M : NT) + 15) / 16;
#pragma unroll 1
      for (int c = 0; c < nchunks; ++c) {
        uint32_t v[16];
        tmem_ld_x16(taddr + 16 * c, v);
        tmem_wait_ld();
        float o[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = __fmul_rn(alpha, __uint_as_float(v[i]));
        if (op != 0) gate_16(o, op, ea, dtb);
        if (g.M <= DIRECT_M) {
          // a few tokens: each warp store is still 64 contiguous bytes
          if (live) {
#pragma unroll
            for (int i = 0; i < DIRECT_M; ++i) {
              if (i >= g.M) break;
              const int64_t at = static_cast<int64_t>(i) * g.ldy + n;
              if (g.out_fp32)
                static_cast<float*>(g.y)[at] = o[i];
              else
                static_cast<__nv_bfloat16*>(g.y)[at] = __float2bfloat16_rn(o[i]);
            }
          }
        } else if (g.out_fp32) {
#pragma unroll
          for (int i = 0; i < 16; ++i) t32[(16 * c + i) * BW + r] = o[i];
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) t16[(16 * c + i) * BW + r] = __float2bfloat16_rn(o[i]);
        }
      }
    } else {
      if (!*abort_flag) record_error(SITE_EPI_TMEM_FULL, warp);
      *abort_flag = 1;
    }
    // all four epilogue warps pass this barrier exactly once, whatever their wait returned
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (ok && !*abort_flag && g.M > DIRECT_M) {
      const int64_t n0 = static_cast<int64_t>(wt) * BW;
      const int esz = g.out_fp32 ? 4 : 2;
      const int chunks = BW * esz / 16;                 // 16-byte chunks per token row
      const int per = 16 / esz;                         // columns per chunk
      const int rows = g.M < NT ? g.M : NT;
      for (int idx = r; idx < rows * chunks; idx += 128) {
        const int j = idx / chunks, c = idx - j * chunks;
        const int64_t col = n0 + c * per;
        if (col < g.N) {                                // N % 16 == 0: chunks are whole
          const uint4 val = *reinterpret_cast<const uint4*>(smem + (j * BW + c * per) * esz);
          char* dst = static_cast<char*>(g.y) + (static_cast<int64_t>(j) * g.ldy + col) * esz;
          *reinterpret_cast<uint4*>(dst) = val;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace nvfp4
