// mk_chunk.cuh -- the gated delta rule over a prompt chunk in chunkwise-
// parallel form (Yang, Kautz & Hatamizadeh, "Gated Delta Networks", ICLR
// 2025: the WY / UT representation of a chunk of delta-rule updates; the
// post "OS Megakernel that match M5 Max Tok/w at 2x the Throughput on RTX
// 3090" reports prompt processing (pp520) beside decode).
//
// Per head, with the state S (dv x dk, o = S q) before a chunk of C
// positions, gates beta_t, alpha_t and cumulative log decay
// g_t = sum_{i<=t} log alpha_i (gamma_t = exp(g_t)), the recurrence
//   S_t = alpha_t S_{t-1} + u_t k_t^T,   u_t = beta_t (v_t - alpha_t S_{t-1} k_t)
// unrolls to  S_t = gamma_t S_0 + sum_{i<=t} exp(g_t - g_i) u_i k_i^T  and
//   (I + L) U = diag(beta) (V - diag(gamma) K S_0^T),
//   L_{t,i} = beta_t exp(g_t - g_i) k_t.k_i  (i < t),
// so with T = (I + L)^-1:
//   U = T diag(beta) V - (T diag(beta gamma) K) S_0^T = Uv - W S_0^T
//   O = diag(gamma) Q S_0^T + (M o Q K^T) U,   M_{t,i} = exp(g_t - g_i) (i <= t)
//   S_C = gamma_C S_0 + U^T diag(exp(g_C - g_t)) K.
// Everything but the three products with S_0 depends on the chunk's inputs
// only: chunk_prep_kernel computes T, W, Uv, diag(gamma) Q, the decayed keys
// and the masked score matrix for every (head, chunk) in parallel;
// chunk_scan_kernel then walks the chunks in order for a slice of state rows
// (rows of S are independent given the shared k, q, gates).  All fp32 on
// CUDA cores: the products are small and the state must stay within 1e-3 of
// the position-by-position recurrence.
#pragma once
#include "mk_ptx.cuh"

namespace mk {
namespace ck {

constexpr int C = 64;            // positions per chunk
constexpr int PREP_THREADS = 256;
constexpr int SCAN_THREADS = 256;
constexpr int SCAN_ROWS = 16;    // state rows per scan block

// Per (head, chunk) block of the prepared operands, in floats:
//   W [C][DK], Uv [C][DV], Qg [C][DK], Kd [C][DK], P [C][C], gammaC (+ pad)
template <int DK>
struct Blk {
  static constexpr int W = 0;
  static constexpr int UV = C * DK;
  static constexpr int QG = 2 * C * DK;
  static constexpr int KD = 3 * C * DK;
  static constexpr int P = 4 * C * DK;
  static constexpr int GC = 4 * C * DK + C * C;
  static constexpr int FLOATS = GC + 4;
};

template <int DK>
constexpr size_t prep_smem() {
  // K, Q, V [C][DK + 1]; L and T [C][C + 1]; g, beta, beta * gamma [C]
  return size_t(3 * C * (DK + 1) + 2 * C * (C + 1) + 3 * C) * 4;
}

// One CTA per (chunk, head).  QK [nh][T][2 DK] (normalised q | k), BAK
// [nh][T] {beta, alpha, -, -}, v of position t, head h, row r at
// V[t * v_ts + h * v_hs + r].  Positions past T are identity steps
// (beta 0, alpha 1).
template <int DK>
__global__ void __launch_bounds__(PREP_THREADS) chunk_prep_kernel(
    const float* __restrict__ QK, const float4* __restrict__ BAK, const float* __restrict__ V,
    size_t v_ts, size_t v_hs, int T, float* __restrict__ out) {
  extern __shared__ __align__(16) float sm[];
  constexpr int LD = DK + 1, LC = C + 1;
  float* Ks = sm;
  float* Qs = Ks + C * LD;
  float* Vs = Qs + C * LD;
  float* Ls = Vs + C * LD;  // L, then reused for W's right factor
  float* Ts = Ls + C * LC;
  float* g = Ts + C * LC;
  float* bt = g + C;
  float* bg = bt + C;
  const int c = blockIdx.x, h = blockIdx.y, nc = gridDim.x, tid = threadIdx.x;
  const int t0 = c * C, n = min(C, T - t0);
  const float* qk = QK + (size_t(h) * T + t0) * 2 * DK;
  for (int i = tid; i < C * DK; i += PREP_THREADS) {
    const int t = i / DK, d = i % DK;
    const bool in = t < n;
    Qs[t * LD + d] = in ? qk[size_t(t) * 2 * DK + d] : 0.f;
    Ks[t * LD + d] = in ? qk[size_t(t) * 2 * DK + DK + d] : 0.f;
    Vs[t * LD + d] = in ? V[size_t(t0 + t) * v_ts + size_t(h) * v_hs + d] : 0.f;
  }
  if (tid < C) {
    const bool in = tid < n;
    const float4 b = in ? BAK[size_t(h) * T + t0 + tid] : make_float4(0.f, 1.f, 0.f, 0.f);
    bt[tid] = b.x;
    // log alpha, bounded below so that a decay that underflows to 0 keeps
    // every difference of cumulative sums finite (exp(-60) ~ 1e-26)
    g[tid] = fmaxf(logf(b.y), -60.f);
  }
  __syncthreads();
  if (tid == 0)
    for (int t = 1; t < C; ++t) g[t] += g[t - 1];  // inclusive prefix sums
  __syncthreads();
  if (tid < C) bg[tid] = bt[tid] * expf(g[tid]);
  // L (strictly lower) and the masked scores P, one entry per thread-step
  float* Pout = out + (size_t(h) * nc + c) * Blk<DK>::FLOATS + Blk<DK>::P;
  for (int e = tid; e < C * C; e += PREP_THREADS) {
    const int t = e / C, i = e % C;
    float kk = 0.f, qk_ = 0.f;
    if (i <= t) {
      for (int d = 0; d < DK; ++d) {
        kk = fmaf(Ks[t * LD + d], Ks[i * LD + d], kk);
        qk_ = fmaf(Qs[t * LD + d], Ks[i * LD + d], qk_);
      }
    }
    const float dec = i <= t ? expf(g[t] - g[i]) : 0.f;
    Ls[t * LC + i] = i < t ? bt[t] * dec * kk : 0.f;
    Pout[e] = i <= t ? dec * qk_ : 0.f;
  }
  __syncthreads();
  // T = (I + L)^-1 by forward substitution, one column per group of four
  // threads (a column depends only on itself): T[t][j] = [t == j] -
  // sum_{j<=i<t} L[t][i] T[i][j]
  {
    const int j = tid >> 2, part = tid & 3;
    for (int t = 0; t < C; ++t) {
      float acc = 0.f;
      if (t > j)
        for (int i = j + part; i < t; i += 4) acc = fmaf(Ls[t * LC + i], Ts[i * LC + j], acc);
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      if (part == 0) Ts[t * LC + j] = t < j ? 0.f : (t == j ? 1.f : -acc);
      __syncwarp();
    }
  }
  __syncthreads();
  // W = T diag(beta gamma) K,  Uv = T diag(beta) V,  Qg = diag(gamma) Q,
  // Kd = diag(exp(g_last - g_t)) K
  float* blk = out + (size_t(h) * nc + c) * Blk<DK>::FLOATS;
  const float glast = g[C - 1];
  for (int e = tid; e < C * DK; e += PREP_THREADS) {
    const int t = e / DK, d = e % DK;
    float w = 0.f, u = 0.f;
    for (int i = 0; i <= t; ++i) {
      const float ti = Ts[t * LC + i];
      w = fmaf(ti * bg[i], Ks[i * LD + d], w);
      u = fmaf(ti * bt[i], Vs[i * LD + d], u);
    }
    blk[Blk<DK>::W + e] = w;
    blk[Blk<DK>::UV + e] = u;
    blk[Blk<DK>::QG + e] = expf(g[t]) * Qs[t * LD + d];
    blk[Blk<DK>::KD + e] = expf(glast - g[t]) * Ks[t * LD + d];
  }
  if (tid == 0) blk[Blk<DK>::GC] = expf(glast);
}

template <int DK>
constexpr size_t scan_smem() {
  // W, Qg, Kd [C][DK]; P [C][C]; Uv [C][R]; U, Oa [C][R]; S [R][DK + 1]
  return size_t(3 * C * DK + C * C + 3 * C * SCAN_ROWS + SCAN_ROWS * (DK + 1) + 4) * 4;
}

// One CTA per (row slice of SCAN_ROWS rows, head): the chunks in order.  S
// [nh][DK][DK] updated in place; O[t * o_ts + h * o_hs + r] receives o.
template <int DK>
__global__ void __launch_bounds__(SCAN_THREADS, 1) chunk_scan_kernel(
    float* __restrict__ S, const float* __restrict__ prep, int T, float* __restrict__ O,
    size_t o_ts, size_t o_hs) {
  extern __shared__ __align__(16) float sm[];
  constexpr int R = SCAN_ROWS, LS = DK + 1;
  float* Ws = sm;
  float* Qg = Ws + C * DK;
  float* Kd = Qg + C * DK;
  float* Ps = Kd + C * DK;
  float* Uv = Ps + C * C;
  float* Us = Uv + C * R;
  float* Oa = Us + C * R;
  float* Ss = Oa + C * R;
  float* gC = Ss + R * LS;
  const int rs = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int r0 = rs * R, nc = (T + C - 1) / C;
  float* Sg = S + (size_t(h) * DK + r0) * DK;
  for (int i = tid; i < R * DK; i += SCAN_THREADS) Ss[(i / DK) * LS + (i % DK)] = Sg[i];
  // thread -> (row r, positions t = tq, tq + 16, tq + 32, tq + 48) for U / O
  const int r = tid % R, tq = tid / R;
  for (int c = 0; c < nc; ++c) {
    const float* blk = prep + (size_t(h) * nc + c) * Blk<DK>::FLOATS;
    __syncthreads();  // the previous chunk's operands are consumed
    for (int i = tid; i < C * DK / 4; i += SCAN_THREADS) {
      reinterpret_cast<float4*>(Ws)[i] = reinterpret_cast<const float4*>(blk + Blk<DK>::W)[i];
      reinterpret_cast<float4*>(Qg)[i] = reinterpret_cast<const float4*>(blk + Blk<DK>::QG)[i];
      reinterpret_cast<float4*>(Kd)[i] = reinterpret_cast<const float4*>(blk + Blk<DK>::KD)[i];
    }
    for (int i = tid; i < C * C / 4; i += SCAN_THREADS)
      reinterpret_cast<float4*>(Ps)[i] = reinterpret_cast<const float4*>(blk + Blk<DK>::P)[i];
    for (int i = tid; i < C * R; i += SCAN_THREADS)
      Uv[i] = blk[Blk<DK>::UV + (i / R) * DK + r0 + (i % R)];
    if (tid == 0) gC[0] = blk[Blk<DK>::GC];
    __syncthreads();
    // U = Uv - W S^T and Oa = Qg S^T for this thread's (t, r) pairs
#pragma unroll
    for (int k = 0; k < C / (SCAN_THREADS / R); ++k) {
      const int t = tq + k * (SCAN_THREADS / R);
      float wu = 0.f, qo = 0.f;
#pragma unroll 8
      for (int d = 0; d < DK; ++d) {
        const float sv = Ss[r * LS + d];
        wu = fmaf(Ws[t * DK + d], sv, wu);
        qo = fmaf(Qg[t * DK + d], sv, qo);
      }
      Us[t * R + r] = Uv[t * R + r] - wu;
      Oa[t * R + r] = qo;
    }
    __syncthreads();
    // O = Oa + (M o Q K^T) U for positions inside T
#pragma unroll
    for (int k = 0; k < C / (SCAN_THREADS / R); ++k) {
      const int t = tq + k * (SCAN_THREADS / R);
      float o = Oa[t * R + r];
      for (int i = 0; i <= t; ++i) o = fmaf(Ps[t * C + i], Us[i * R + r], o);
      if (c * C + t < T) O[size_t(c * C + t) * o_ts + size_t(h) * o_hs + r0 + r] = o;
    }
    // S <- gamma_C S + U^T Kd: thread -> row tid / 16, columns (tid % 16) + 16 j
    {
      const int sr = tid / (SCAN_THREADS / R), sc = tid % (SCAN_THREADS / R);
      const float gc = gC[0];
#pragma unroll
      for (int j = 0; j < DK / (SCAN_THREADS / R); ++j) {
        const int d = sc + j * (SCAN_THREADS / R);
        float acc = gc * Ss[sr * LS + d];
#pragma unroll 8
        for (int t = 0; t < C; ++t) acc = fmaf(Us[t * R + sr], Kd[t * DK + d], acc);
        // every read of Ss for this chunk happened before the barrier above
        Ss[sr * LS + d] = acc;
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < R * DK; i += SCAN_THREADS) Sg[i] = Ss[(i / DK) * LS + (i % DK)];
}

// q, k [heads][T][DK] -> QK [heads][T][2 DK]; alpha, beta [heads][T] -> BAK
// (the layout the prompt path's preparation kernel writes).
template <int DK>
__global__ void chunk_pack_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                  const float* __restrict__ alpha, const float* __restrict__ beta,
                                  size_t n_pos, float* __restrict__ QK, float4* __restrict__ BAK) {
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n_pos * DK;
       i += size_t(gridDim.x) * blockDim.x) {
    const size_t p = i / DK, d = i % DK;
    QK[p * 2 * DK + d] = q[i];
    QK[p * 2 * DK + DK + d] = k[i];
    if (d == 0) BAK[p] = make_float4(beta[p], alpha[p], 0.f, 0.f);
  }
}

}  // namespace ck
}  // namespace mk
