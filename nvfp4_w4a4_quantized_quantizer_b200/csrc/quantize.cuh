// quantize.cuh -- NVFP4 quantisation kernels (HBM-bound).
//
// k_quantize: bf16 rows -> packed E2M1 codes + UE4M3 block scales written
// directly in the 128x4 atom layout that tcgen05 block-scaled MMA consumes.
// The arithmetic is the NVFP4 16-element block scaling of the paper "Why
// Gated DeltaNet Survives 4-Bit Quantization" (bayesiansapien wiki, "The
// four-part mechanism study", part 1), with these steps per block:
//   c     = fp32(6 * gs)
//   s     = E4M3_RNE_satfinite(fp32(amax16 / c))
//   r     = fp32(1 / fp32(s_dec * gs))       (0 when s_dec == 0)
//   q_k   = E2M1_RNE_satfinite(fp32(x_k * r))
// Every rounding is an explicit _rn intrinsic or a .rn conversion, so the
// compiler cannot contract or reorder it.
//
// Work mapping: a warp work unit is (row, 1024-element segment), streamed
// into shared memory by a bulk copy (see "Staging" below); lane t owns one
// whole 16-element block per 512 elements, writes its 8 code bytes (the
// warp writes 256 contiguous bytes), and every 4th lane gathers the scale
// bytes of blocks j..j+3 (contiguous in the atom layout) into one 32-bit
// store.  The block reciprocal r depends only on the scale code, so the
// launch carries the 128-entry table r[s] = fp32(1 / fp32(s_dec * gs)) (0 for
// s = 0), computed on the host with IEEE fp32 arithmetic — the same rounding
// as the device reciprocal — instead of a decode, a multiply and a
// reciprocal per block.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace nvfp4 {

// ------------------------------------------------------------ conversions
// Eight fp32 values -> eight E2M1 codes packed in 32 bits, element e in
// bits 4e..4e+3 (even elements in the low nibble of each byte).  The PTX
// conversion puts its first source in the high nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// fp32 (>= 0) -> unsigned E4M3 code, round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t cvt_e4m3(float v) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
  return static_cast<uint32_t>(out) & 0xFFu;
}

// Unsigned E4M3 code -> its exact fp32 value, built from the bit fields.
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const uint32_t e = (code >> 3) & 0xFu;
  const uint32_t m = code & 7u;
  if (e == 0) return static_cast<float>(m) * 0.001953125f;  // m * 2^-9, exact
  return __uint_as_float(((e + 120u) << 23) | (m << 20));   // (1 + m/8) * 2^(e-7)
}

// Byte offset of logical scale S[r, j] inside the 128x4 atom layout.
__host__ __device__ __forceinline__ uint64_t sf_offset(int64_t r, int64_t j, int64_t K) {
  const int64_t kb4 = K / 64;  // atoms per 128-row block along K
  return static_cast<uint64_t>(((r >> 7) * kb4 + (j >> 2)) * 512 + (r & 31) * 16 +
                               ((r >> 5) & 3) * 4 + (j & 3));
}

struct QuantArgs {
  const __nv_bfloat16* x;  // first row of the range
  int64_t rows;            // rows in the range
  int64_t K;
  int64_t ldx;             // elements
  int64_t row0;            // logical row of x[0] in the code / scale buffers
  float gs;
  uint8_t* codes;          // base of the full code buffer [*, K/2]
  uint8_t* scales;         // base of the full scale buffer (atom layout)
  int64_t pad_from;        // zero scale rows [pad_from, pad_to)
  int64_t pad_to;
  uint64_t wait_ns;        // bound on each wait for a staged copy
  float rtab[128];         // fp32(1 / fp32(e4m3(s) * gs)), 0 for s == 0
};

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Staging: every warp owns a ring of QUANT_SLOTS shared-memory slots and
// streams its work units into them with cp.async.bulk (one contiguous copy
// of a row segment per unit, completion counted on the slot's mbarrier), so
// each SM keeps ~QUANT_SLOTS x 2 KB x (resident warps) bytes of HBM reads in
// flight independent of registers; the warp then quantises the unit out of
// shared memory and refills the slot with its unit QUANT_SLOTS ahead.
constexpr int QUANT_THREADS = 256;
constexpr int QUANT_WARPS = QUANT_THREADS / 32;
constexpr int QUANT_UNIT = 1024;                 // elements per work unit (2 KB of bf16)
constexpr int QUANT_SLOTS = 4;
constexpr int QUANT_SMEM = QUANT_WARPS * QUANT_SLOTS * QUANT_UNIT * 2;   // 64 KB
constexpr int QUANT_BAR_BYTES = QUANT_WARPS * QUANT_SLOTS * 8;

// |x| max of sixteen bf16 values (eight packed words), exact.  max with
// .xorsign.abs compares magnitudes (bf16 comparisons are exact, subnormals
// kept) and returns the larger magnitude with a sign we discard; the word
// order does not matter.  The result is the bf16 magnitude as fp32 bits.
__device__ __forceinline__ uint32_t max_abs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ float bf16x16_absmax(const uint32_t (&w)[8]) {
  const uint32_t m01 = max_abs_bf16x2(w[0], w[1]);
  const uint32_t m23 = max_abs_bf16x2(w[2], w[3]);
  const uint32_t m45 = max_abs_bf16x2(w[4], w[5]);
  const uint32_t m67 = max_abs_bf16x2(w[6], w[7]);
  const uint32_t m = max_abs_bf16x2(max_abs_bf16x2(m01, m23), max_abs_bf16x2(m45, m67));
  const uint32_t both = max_abs_bf16x2(m, __byte_perm(m, 0u, 0x1032));   // both halves = the max
  return __uint_as_float((both & 0x7FFFu) << 16);
}

// The two bf16 values of a packed word times r, as two fp32 products each
// rounded to nearest (one packed fp32 multiply; no flush of subnormals).
__device__ __forceinline__ void bf16x2_times(uint32_t w, uint64_t rr, float& lo, float& hi) {
  uint64_t x, d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(w << 16), "r"(w & 0xFFFF0000u));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(x), "l"(rr));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(d));
}

// Position of a warp's current work unit (row, unit within the row).  A warp
// visits units gwarp, gwarp + nwarps, ...; the cursor advances by nwarps
// without a division (nwarps = step_rows * per_row + step_cols).
struct UnitCursor {
  int64_t row;
  int col;       // unit index within the row
  __device__ __forceinline__ void advance(int64_t step_rows, int step_cols, int per_row) {
    row += step_rows;
    col += step_cols;
    if (col >= per_row) {
      col -= per_row;
      ++row;
    }
  }
};

__global__ void __launch_bounds__(QUANT_THREADS) k_quantize(const __grid_constant__ QuantArgs a) {
  extern __shared__ __align__(128) uint8_t qsmem[];
  // The reciprocal table in shared memory: the lanes of a warp look up
  // different scale codes, which a constant-bank (parameter) load would
  // serve one distinct address at a time.
  __shared__ float s_rtab[128];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  for (int t = threadIdx.x; t < 128; t += QUANT_THREADS) s_rtab[t] = a.rtab[t];
  __syncthreads();
  uint8_t* ring = qsmem + warp * (QUANT_SLOTS * QUANT_UNIT * 2);
  uint64_t* bars = reinterpret_cast<uint64_t*>(qsmem + QUANT_SMEM) + warp * QUANT_SLOTS;
  const int K = static_cast<int>(a.K);
  const int per_row = (K + QUANT_UNIT - 1) / QUANT_UNIT;
  const int64_t units = a.rows * per_row;
  const int64_t gwarp = static_cast<int64_t>(blockIdx.x) * QUANT_WARPS + warp;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * QUANT_WARPS;
  const float c = __fmul_rn(6.0f, a.gs);
  const int64_t code_ld = a.K / 2;
  const int64_t kb4 = a.K / 64;                  // scale atoms per 128-row block along K
  const uint64_t pol = policy_evict_first();
  const int64_t step_rows = nwarps / per_row;
  const int step_cols = static_cast<int>(nwarps - step_rows * per_row);

  // With launch overlap this grid may start before the kernel ahead of it
  // has finished: let the kernel behind it be scheduled, then wait before
  // reading x or writing codes and scales.
  griddep_launch_dependents();
  griddep_wait();

  if (lane == 0) {
    for (int s = 0; s < QUANT_SLOTS; ++s) mbar_init(smem_addr(bars + s), 1);
    fence_mbar_init();
  }
  __syncwarp();
  // lane 0 starts the copy of unit `at` (the warp's i-th) into slot i % QUANT_SLOTS
  UnitCursor at{gwarp / per_row, static_cast<int>(gwarp % per_row)};
  auto issue = [&](int64_t i) {
    if (at.row >= a.rows) return;
    const int col = at.col * QUANT_UNIT;
    const uint32_t bytes = static_cast<uint32_t>(min(QUANT_UNIT, K - col)) * 2u;
    const int s = static_cast<int>(i % QUANT_SLOTS);
    mbar_arrive_expect_tx(smem_addr(bars + s), bytes);
    bulk_load(smem_addr(ring + s * (QUANT_UNIT * 2)), a.x + at.row * a.ldx + col, bytes,
              smem_addr(bars + s), pol);
    at.advance(step_rows, step_cols, per_row);
  };
  if (lane == 0)
    for (int i = 0; i < QUANT_SLOTS; ++i) issue(i);

  UnitCursor cur{gwarp / per_row, static_cast<int>(gwarp % per_row)};
  int64_t i = 0;
  bool ok = true;
  for (; cur.row < a.rows; cur.advance(step_rows, step_cols, per_row), ++i) {
    const int s = static_cast<int>(i % QUANT_SLOTS);
    if (!mbar_wait_warp(smem_addr(bars + s), static_cast<uint32_t>((i / QUANT_SLOTS) & 1), a.wait_ns,
                   nullptr)) {
      if (lane == 0) record_error(SITE_QUANT, static_cast<uint32_t>(warp));
      ok = false;
      break;
    }
    const int col = cur.col * QUANT_UNIT;
    const int n = min(QUANT_UNIT, K - col);
    const int64_t grow = a.row0 + cur.row;
    const uint32_t slot = smem_addr(ring + s * (QUANT_UNIT * 2));
    // this unit's code row and the scale bytes of its first 4-block group
    uint8_t* code_row = a.codes + grow * code_ld + col / 2;
    uint8_t* sf_unit = a.scales + ((grow >> 7) * kb4 + col / 64) * 512 + (grow & 31) * 16 +
                       ((grow >> 5) & 3) * 4;
#pragma unroll
    for (int p = 0; p < QUANT_UNIT / 512; ++p) {
      const int e0 = p * 512;
      if (e0 >= n) break;                                 // warp-uniform
      const int e = e0 + lane * 16;                       // this lane's block
      const bool live = e < n;                            // uniform per 4 lanes (n % 64 == 0)
      uint32_t w[8];
      // lanes 4..7 of each group of 8 read their halves in the other order,
      // so a quarter-warp's 16-byte reads cover all 32 banks once
      const uint32_t h = static_cast<uint32_t>((lane >> 2) & 1) * 16u;
      const uint4 v0 = ld_shared_v4(slot + e * 2 + h);
      const uint4 v1 = ld_shared_v4(slot + e * 2 + (h ^ 16u));
      // w holds the block's two halves in load order (swapped for h != 0):
      // the amax does not depend on the order, the code words are put back
      // in element order before the store
      w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
      w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
      const float amax = bf16x16_absmax(w);
      const uint32_t sc = cvt_e4m3(__fdiv_rn(amax, c));
      const float rr = s_rtab[sc];
      uint64_t rr2;
      asm("mov.b64 %0, {%1, %1};" : "=l"(rr2) : "f"(rr));
      float f[8];
      uint32_t qv[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
        for (int k = 0; k < 4; ++k) bf16x2_times(w[4 * hh + k], rr2, f[2 * k], f[2 * k + 1]);
        qv[hh] = cvt_e2m1x8(f);
      }
      if (sc == 0) qv[0] = qv[1] = 0u;
      // scale bytes of blocks 4g..4g+3 (lanes 4g..4g+3) -> lane 4g
      const uint32_t s1 = __shfl_down_sync(0xffffffffu, sc, 1);
      const uint32_t s2 = __shfl_down_sync(0xffffffffu, sc, 2);
      const uint32_t s3 = __shfl_down_sync(0xffffffffu, sc, 3);
      if (live) {
        *reinterpret_cast<uint2*>(code_row + e / 2) = h ? make_uint2(qv[1], qv[0]) : make_uint2(qv[0], qv[1]);
        if ((lane & 3) == 0) {
          // blocks e/16 .. e/16 + 3 of the unit: atom (e / 64) after the unit's first
          const uint32_t word = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
          *reinterpret_cast<uint32_t*>(sf_unit + (e / 64) * 512) = word;
        }
      }
    }
    // every lane's reads of the slot are done (their results are stored);
    // order them before the bulk copy that refills it
    __syncwarp();
    if (lane == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(i + QUANT_SLOTS);
    }
  }
  // copies still in flight (only after a failed wait) must land before exit
  if (!ok && lane == 0) {
    for (int64_t j = i; j < i + QUANT_SLOTS; ++j) {
      if (gwarp + j * nwarps >= units) break;
      mbar_wait(smem_addr(bars + (j % QUANT_SLOTS)), static_cast<uint32_t>((j / QUANT_SLOTS) & 1),
                a.wait_ns, nullptr);
    }
  }

  // zero the scale bytes of the padding rows (rows past the last real row
  // inside the last 128-row block)
  const int64_t kb = a.K / 16;
  const int64_t pad_words = (a.pad_to - a.pad_from) * (kb / 4);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * QUANT_THREADS + threadIdx.x; t < pad_words;
       t += static_cast<int64_t>(gridDim.x) * QUANT_THREADS) {
    const int64_t r = a.pad_from + t / (kb / 4);
    const int64_t j = (t % (kb / 4)) * 4;
    *reinterpret_cast<uint32_t*>(a.scales + sf_offset(r, j, a.K)) = 0u;
  }
}

// ------------------------------------------------------------------- amax
// out[0] = max |x| over rows x K.  `out` must hold 0.0f on entry (the host
// clears it on the same stream); non-negative floats order like their bit
// patterns, so an integer atomicMax on the bits is an exact float max.
constexpr int AMAX_THREADS = 256;

__global__ void __launch_bounds__(AMAX_THREADS) k_amax(const __nv_bfloat16* __restrict__ x,
                                                       int64_t rows, int64_t K, int64_t ldx,
                                                       float* out) {
  const int lane = threadIdx.x & 31;
  const int64_t gwarp = (static_cast<int64_t>(blockIdx.x) * AMAX_THREADS + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * AMAX_THREADS) >> 5;
  float m = 0.0f;
  for (int64_t r = gwarp; r < rows; r += nwarps) {
    const __nv_bfloat16* p = x + r * ldx;
    for (int64_t k = lane * 8; k < K; k += 256) {
      float f[8];
      bf16x8_to_f32(ld_stream_v4(p + k), f);
#pragma unroll
      for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float red[AMAX_THREADS / 32];
  if (lane == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.0f;
    for (int i = 0; i < AMAX_THREADS / 32; ++i) b = fmaxf(b, red[i]);
    atomicMax(reinterpret_cast<unsigned int*>(out), __float_as_uint(b));
  }
}

// ------------------------------------------------------- MLP glue (SiLU*up)
// h = fp32(silu(g) * u) for bf16-valued g and u: g / (1 + e^-g) with an
// IEEE divide, then the product, each step rounded to nearest and none
// contracted (the fused gate_up epilogue computes the same function, so
// both paths give identical h).
__device__ __forceinline__ float silu_mul_f32(float g, float u) {
  return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), u);
}

// Block reciprocal of scale code `code` under global scale gs:
// fp32(1 / fp32(e4m3(code) * gs)), 0 for code 0 -- the entry of k_quantize's
// host-built table, computed on the device with the same two roundings.
__device__ __forceinline__ float block_reciprocal(uint32_t code, float gs) {
  return code == 0 ? 0.0f : __frcp_rn(__fmul_rn(e4m3_value(code), gs));
}

constexpr int SILU_THREADS = 256;

__global__ void __launch_bounds__(SILU_THREADS) k_silu_mul(const __nv_bfloat16* __restrict__ gu,
                                                           int64_t M, int64_t H, int64_t ld_in,
                                                           __nv_bfloat16* __restrict__ h,
                                                           int64_t ld_out) {
  const int64_t vec_per_row = H / 8;
  const int64_t total = M * vec_per_row;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * SILU_THREADS + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * SILU_THREADS) {
    const int64_t m = t / vec_per_row;
    const int64_t j = (t - m * vec_per_row) * 8;
    float g[8], u[8];
    bf16x8_to_f32(ld_stream_v4(gu + m * ld_in + j), g);
    bf16x8_to_f32(ld_stream_v4(gu + m * ld_in + H + j), u);
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a0 = silu_mul_f32(g[2 * e], u[2 * e]);
      const float a1 = silu_mul_f32(g[2 * e + 1], u[2 * e + 1]);
      const __nv_bfloat162 p = __floats2bfloat162_rn(a0, a1);
      w[e] = *reinterpret_cast<const uint32_t*>(&p);
    }
    *reinterpret_cast<uint4*>(h + m * ld_out + j) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ------------------------------------------------------ FP8 (E4M3) KV cache
// The pages' other shipped recipe: KV-cache tensors in FP8 E4M3 under a
// calibrated per-tensor scale.  code = sign | E4M3_RNE_satfinite(fp32(x * r))
// with r = fp32(1 / scale) formed on the host; eight bf16 in (16 bytes),
// eight codes out (8 bytes) per thread and step.  HBM-bound.
constexpr int KV_THREADS = 256;

// Two fp32 values -> two E4M3 codes, a in the low byte (the PTX conversion
// puts its first source in the high byte).
__device__ __forceinline__ uint32_t cvt_e4m3x2(float a, float b) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(b), "f"(a));
  return static_cast<uint32_t>(out);
}

__global__ void __launch_bounds__(KV_THREADS) k_kv_fp8(const __nv_bfloat16* __restrict__ x,
                                                       int64_t n8, float r,
                                                       uint2* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * KV_THREADS + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * KV_THREADS) {
    float f[8];
    bf16x8_to_f32(ld_stream_v4(x + i * 8), f);
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
      w[h] = cvt_e4m3x2(__fmul_rn(f[4 * h], r), __fmul_rn(f[4 * h + 1], r)) |
             (cvt_e4m3x2(__fmul_rn(f[4 * h + 2], r), __fmul_rn(f[4 * h + 3], r)) << 16);
    out[i] = make_uint2(w[0], w[1]);
  }
}

// ------------------------------------------------------------ test kernels
__global__ void k_test_e2m1(const float* in, uint8_t* out, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
  {
    const float v[8] = {in[i], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    out[i] = static_cast<uint8_t>(cvt_e2m1x8(v) & 0xFu);
  }
}

__global__ void k_test_e4m3(const float* in, uint8_t* out, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = static_cast<uint8_t>(cvt_e4m3(in[i]));
}

// One CTA waits on an mbarrier that nothing arrives on; the bounded wait
// must give up after limit_ns and record the error word.
__global__ void k_test_wait_timeout(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait(smem_addr(&bar), 0, limit_ns, &abort_flag)) record_error(SITE_TEST, 0);
  }
  __syncthreads();
}

}  // namespace nvfp4
