// gdn.cuh -- the Gated DeltaNet state recurrence (the step after the GDN
// in-projection), chunk by chunk.
//
// The recurrent half of the hybrid model keeps, per value head, a state
// S in R^{dv x dk} that every token overwrites along its key direction
// (bayesiansapien wiki, "The four-part mechanism study", part 3; the
// formula is the published gated delta rule):
//   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t,
// with alpha_t = exp(g_t) (g and beta from the in-projection's gate
// epilogue) and unit keys.  Per chunk of C tokens starting from S_0, with
// G_t the running sum of g inside the chunk:
//   A_tj = beta_t e^{G_t - G_j} (k_t . k_j)               (j < t)
//   (I + A) U = diag(beta) V - diag(beta e^G) K S_0^T      (forward substitution)
//   O_t = e^{G_t} S_0 q_t + sum_{j <= t} e^{G_t - G_j} (q_t . k_j) U_j
//   S_C = e^{G_C} S_0 + sum_t e^{G_C - G_t} U_t k_t^T
//
// Each value row of S evolves on its own (S_i <- alpha S_i (I - beta k k^T)
// + beta v_i k^T reads only the keys, beta and g), so a head splits across
// CTAs by value rows; only the key products (A, and Q K^T) are computed by
// every CTA of the head.
//
// k_gdn_chunked: one CTA per (value head, block of value rows); the fp32
// state rows and one chunk's keys, queries and value columns stay in shared
// memory (at most 191 KB); fp32 CUDA-core arithmetic with register tiles fed
// by 128-bit shared loads.  The products are dense and would belong on the
// tensor cores.
#pragma once

#include <cstdint>

namespace nvfp4 {
namespace gdn {
constexpr int C = 64;          // tokens per chunk
constexpr int D = 128;         // key and value head width
// Rows of S, K and Q are padded to 132 floats: 16-byte aligned for float4
// loads along d, and 33 16-byte bank groups apart, so eight lanes reading
// eight consecutive rows at one d (a quarter warp's 128-bit access) hit
// eight different groups.
constexpr int LD = D + 4;
constexpr int CP = C + 4;      // padded rows of A: 16-byte aligned, 17 bank groups apart
constexpr int THREADS = 256;
constexpr int SMEM_FLOATS = D * LD + 2 * C * LD + C * D + C * CP + 4 * C + C * 16;
constexpr int SMEM_BYTES = SMEM_FLOATS * 4;
static_assert(SMEM_BYTES <= 232448, "shared memory");
}  // namespace gdn

struct GdnArgs {
  const float* q;      // [T, Hk, D] (unit rows expected for k; q as is)
  const float* k;      // [T, Hk, D]
  const float* v;      // [T, Hv, D]
  const float* g;      // [T, Hv] log decay (<= 0)
  const float* beta;   // [T, Hv]
  float* o;            // [T, Hv, D]
  float* state;        // [Hv, D (value), D (key)]: initial state in, final state out
  int64_t T;
  int Hv, group;       // value heads; value heads per key head (Hk = Hv / group)
  int parts;           // CTAs per head, each with rows [p * rows, min(D, (p + 1) * rows))
  int rows;
};

// acc[a][b] = sum_d X[ra[a] * LD + d] * Y[rb[b] * LD + d] over d < D, d in
// order: a 4 x 4 register tile of row dot products, four d at a time from
// 128-bit shared loads (8 loads per 64 FMAs).
__device__ __forceinline__ void dot_tile4(const float* X, const int (&ra)[4], const float* Y,
                                          const int (&rb)[4], float (&acc)[4][4]) {
  using namespace gdn;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
#pragma unroll 2
  for (int d = 0; d < D; d += 4) {
    float4 x[4], y[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = *reinterpret_cast<const float4*>(X + ra[i] * LD + d);
#pragma unroll
    for (int j = 0; j < 4; ++j) y[j] = *reinterpret_cast<const float4*>(Y + rb[j] * LD + d);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[i][j] = fmaf(x[i].x, y[j].x, acc[i][j]);
        acc[i][j] = fmaf(x[i].y, y[j].y, acc[i][j]);
        acc[i][j] = fmaf(x[i].z, y[j].z, acc[i][j]);
        acc[i][j] = fmaf(x[i].w, y[j].w, acc[i][j]);
      }
  }
}

__global__ void __launch_bounds__(gdn::THREADS, 1) k_gdn_chunked(const GdnArgs a) {
  using namespace gdn;
  extern __shared__ __align__(16) float gsm[];
  float* S = gsm;                   // [rn value rows][LD key]
  float* Kc = S + D * LD;           // [C][LD]
  float* Qc = Kc + C * LD;          // [C][LD]
  float* Vc = Qc + C * LD;          // [C][RP]: values, then the right-hand side, then U
  float* A = Vc + C * D;            // [C][CP]: A, then the masked, scaled Q K^T
  float* G = A + C * CP;            // [C] running log decay
  float* B = G + C;                 // [C] beta
  float* E = B + C;                 // [C] e^{G_t}
  float* W = E + C;                 // [C] e^{G_last - G_t}
  float* Ti = W + C;                // [C / 16][16][16] inverses of the 16 x 16 diagonal blocks of I + A
  const int h = blockIdx.x / a.parts;          // value head
  const int r0 = (blockIdx.x % a.parts) * a.rows;
  const int rn = min(D, r0 + a.rows) - r0;      // this CTA's value rows [r0, r0 + rn)
  const int RP = (rn + 3) & ~3;                  // row pitch of Vc: float4 rows, columns past rn zero
  const int hk = h / a.group;
  const int Hk = a.Hv / a.group;
  const int tid = threadIdx.x;
  float* state = a.state + (static_cast<int64_t>(h) * D + r0) * D;

  for (int x = tid; x < rn * D; x += THREADS) S[(x / D) * LD + x % D] = state[x];
  for (int x = tid; x < C * RP; x += THREADS) Vc[x] = 0.0f;

  for (int64_t c0 = 0; c0 < a.T; c0 += C) {
    const int cn = static_cast<int>(a.T - c0 < C ? a.T - c0 : C);
    __syncthreads();   // the previous chunk is done with Kc, Qc, Vc, A and S
    for (int x = tid; x < C * D / 4; x += THREADS) {
      const int t = x / (D / 4), d = 4 * (x - t * (D / 4));
      const bool live = t < cn;
      const int64_t at = (static_cast<int64_t>(c0 + t) * Hk + hk) * D + d;
      const float4 zero = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      *reinterpret_cast<float4*>(Kc + t * LD + d) = live ? *reinterpret_cast<const float4*>(a.k + at) : zero;
      *reinterpret_cast<float4*>(Qc + t * LD + d) = live ? *reinterpret_cast<const float4*>(a.q + at) : zero;
    }
    for (int x = tid; x < C * rn; x += THREADS) {
      const int t = x / rn, i = x - t * rn;
      Vc[t * RP + i] = t < cn ? a.v[((c0 + t) * a.Hv + h) * D + r0 + i] : 0.0f;
    }
    if (tid < 32) {
      // running sum of g over the chunk: 64 values, two per lane
      float g0 = 0.0f, g1 = 0.0f;
      const int t0 = 2 * tid, t1 = 2 * tid + 1;
      if (t0 < cn) g0 = a.g[(c0 + t0) * a.Hv + h];
      if (t1 < cn) g1 = a.g[(c0 + t1) * a.Hv + h];
      float run = g0 + g1;
      for (int off = 1; off < 32; off <<= 1) {
        const float up = __shfl_up_sync(0xffffffffu, run, off);
        if (tid >= off) run += up;
      }
      float before = __shfl_up_sync(0xffffffffu, run, 1);   // sum over earlier pairs
      if (tid == 0) before = 0.0f;
      G[t0] = before + g0;
      G[t1] = G[t0] + g1;
      B[t0] = t0 < cn ? a.beta[(c0 + t0) * a.Hv + h] : 0.0f;
      B[t1] = t1 < cn ? a.beta[(c0 + t1) * a.Hv + h] : 0.0f;
      E[t0] = expf(G[t0]);
      E[t1] = expf(G[t1]);
    }
    __syncthreads();

    // Register tiles of 4 x 4 outputs.  Token rows and key columns map as
    // base + 16 * k (and value rows as 4 * tile + k), so that across a warp
    // the shared loads of the inner loops hit distinct banks or broadcast.
    const int ni = (rn + 3) / 4;              // tiles of 4 value rows
    // A_tj = beta_t e^{G_t - G_j} (k_t . k_j), j < t
    {
      const int ty = tid / 16, tx = tid % 16;
      int rt[4], rj[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        rt[k] = ty + 16 * k;
        rj[k] = tx + 16 * k;
      }
      float acc[4][4];
      dot_tile4(Kc, rt, Kc, rj, acc);
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int t = rt[p], j = rj[q];
          A[t * CP + j] = (j < t && t < cn) ? acc[p][q] * B[t] * expf(G[t] - G[j]) : 0.0f;
        }
    }
    // right-hand side: beta_t v_t - beta_t e^{G_t} S_0 k_t (this CTA's rows)
    for (int tile = tid; tile < 16 * ni; tile += THREADS) {
      const int tt = tile % 16, ti = tile / 16;
      int rt[4], ri[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        rt[k] = tt + 16 * k;
        ri[k] = min(4 * ti + k, rn - 1);
      }
      float acc[4][4];
      dot_tile4(Kc, rt, S, ri, acc);
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int t = rt[p], i = 4 * ti + q;
          if (i < rn) Vc[t * RP + i] = B[t] * Vc[t * RP + i] - B[t] * E[t] * acc[p][q];
        }
    }
    __syncthreads();
    // (I + A) U = rhs in 16-row blocks.  The diagonal blocks of I + A are
    // unit lower triangular and depend on A alone: their inverses are
    // formed once per chunk (one column per thread, 64 threads).  Then for
    // each block: the terms of the rows solved in earlier blocks (one
    // product over all threads), and the block's rows as its inverse times
    // that residual.  Rows past cn have zero right-hand sides and zero rows
    // of A.
    if (tid < C) {
      const int b = tid >> 4, c = tid & 15;
      const float* Ab = A + (16 * b) * CP + 16 * b;      // the diagonal block
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float v = r == c ? 1.0f : 0.0f;
#pragma unroll
        for (int j = 0; j < r; ++j)
          if (j >= c) v = fmaf(-Ab[r * CP + j], x[j], v);
        x[r] = r < c ? 0.0f : v;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) Ti[(b * 16 + r) * 16 + c] = x[r];
    }
    __syncthreads();
    for (int t0 = 0; t0 < cn; t0 += 16) {
      constexpr int PER = (16 * D + THREADS - 1) / THREADS;   // outputs per thread, at most
      if (t0 > 0) {
        for (int x = tid; x < 16 * rn; x += THREADS) {
          const int t = t0 + x / rn, i = x - (x / rn) * rn;
          const float* At = A + t * CP;
          float s0 = 0.0f, s1 = 0.0f;
          for (int j = 0; j < t0; j += 2) {
            s0 = fmaf(At[j], Vc[j * RP + i], s0);
            s1 = fmaf(At[j + 1], Vc[(j + 1) * RP + i], s1);
          }
          Vc[t * RP + i] -= s0 + s1;
        }
        __syncthreads();
      }
      const float* Tb = Ti + (t0 / 16) * 256;
      float u[PER];
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int x = tid + k * THREADS;
        u[k] = 0.0f;
        if (x < 16 * rn) {
          const int r = x / rn, i = x - r * rn;
          float acc = 0.0f;
          for (int c = 0; c <= r; ++c) acc = fmaf(Tb[r * 16 + c], Vc[(t0 + c) * RP + i], acc);
          u[k] = acc;
        }
      }
      __syncthreads();   // the block's residual rows are read
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int x = tid + k * THREADS;
        if (x < 16 * rn) Vc[(t0 + x / rn) * RP + x % rn] = u[k];
      }
      __syncthreads();
    }
    // P_tj = e^{G_t - G_j} (q_t . k_j), j <= t (into A)
    {
      const int ty = tid / 16, tx = tid % 16;
      int rt[4], rj[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        rt[k] = ty + 16 * k;
        rj[k] = tx + 16 * k;
      }
      float acc[4][4];
      dot_tile4(Qc, rt, Kc, rj, acc);
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int t = rt[p], j = rj[q];
          A[t * CP + j] = (j <= t && t < cn) ? acc[p][q] * expf(G[t] - G[j]) : 0.0f;
        }
    }
    __syncthreads();
    // o_t = e^{G_t} S_0 q_t + sum_j P_tj U_j (P_tj = 0 past t)
    for (int tile = tid; tile < 16 * ni; tile += THREADS) {
      const int tt = tile % 16, ti = tile / 16;
      int rt[4], ri[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        rt[k] = tt + 16 * k;
        ri[k] = min(4 * ti + k, rn - 1);
      }
      float sq[4][4];
      dot_tile4(Qc, rt, S, ri, sq);
      float pu[4][4];
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) pu[p][q] = 0.0f;
      // four j at a time: P's entries past a row's own token are zero, and
      // the rows of A and U hold 64 columns and 64 rows
      const int jmax = min(rt[3], cn - 1);     // the tile's last token row
      const int vi = min(4 * ti, RP - 4);      // this tile's four value columns of U
      for (int j = 0; j <= jmax; j += 4) {
        float4 pv[4], uv[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) pv[p] = *reinterpret_cast<const float4*>(A + rt[p] * CP + j);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) uv[jj] = *reinterpret_cast<const float4*>(Vc + (j + jj) * RP + vi);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float pj[4] = {pv[p].x, pv[p].y, pv[p].z, pv[p].w};
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            pu[p][0] = fmaf(pj[jj], uv[jj].x, pu[p][0]);
            pu[p][1] = fmaf(pj[jj], uv[jj].y, pu[p][1]);
            pu[p][2] = fmaf(pj[jj], uv[jj].z, pu[p][2]);
            pu[p][3] = fmaf(pj[jj], uv[jj].w, pu[p][3]);
          }
        }
      }
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int t = rt[p], i = 4 * ti + q;
          if (t < cn && i < rn) a.o[((c0 + t) * a.Hv + h) * D + r0 + i] = E[t] * sq[p][q] + pu[p][q];
        }
    }
    const float gc = G[cn - 1];
    if (tid < C) W[tid] = tid < cn ? expf(gc - G[tid]) : 0.0f;
    __syncthreads();   // every output of the chunk read the old state; W is ready
    // S = e^{G_C} S_0 + sum_t e^{G_C - G_t} U_t k_t^T: a thread updates 4
    // value rows x 8 consecutive key columns (float4 loads of U, K and S)
    const float ec = expf(gc);
    for (int tile = tid; tile < 16 * ni; tile += THREADS) {
      const int tj = tile % 16, ti = tile / 16;
      const int c0k = 8 * tj;
      float acc[4][8];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float4 lo = *reinterpret_cast<const float4*>(S + (4 * ti + p) * LD + c0k);
        const float4 hi = *reinterpret_cast<const float4*>(S + (4 * ti + p) * LD + c0k + 4);
        acc[p][0] = ec * lo.x; acc[p][1] = ec * lo.y; acc[p][2] = ec * lo.z; acc[p][3] = ec * lo.w;
        acc[p][4] = ec * hi.x; acc[p][5] = ec * hi.y; acc[p][6] = ec * hi.z; acc[p][7] = ec * hi.w;
      }
      for (int t = 0; t < cn; ++t) {
        const float w = W[t];
        const float4 u = *reinterpret_cast<const float4*>(Vc + t * RP + 4 * ti);
        const float4 k0 = *reinterpret_cast<const float4*>(Kc + t * LD + c0k);
        const float4 k1 = *reinterpret_cast<const float4*>(Kc + t * LD + c0k + 4);
        const float uv[4] = {u.x * w, u.y * w, u.z * w, u.w * w};
        const float kv[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[p][q] = fmaf(uv[p], kv[q], acc[p][q]);
      }
#pragma unroll
      for (int p = 0; p < 4; ++p)
        if (4 * ti + p < rn) {
          *reinterpret_cast<float4*>(S + (4 * ti + p) * LD + c0k) =
              make_float4(acc[p][0], acc[p][1], acc[p][2], acc[p][3]);
          *reinterpret_cast<float4*>(S + (4 * ti + p) * LD + c0k + 4) =
              make_float4(acc[p][4], acc[p][5], acc[p][6], acc[p][7]);
        }
    }
  }
  __syncthreads();
  for (int x = tid; x < rn * D; x += THREADS) state[x] = S[(x / D) * LD + x % D];
}

}  // namespace nvfp4
