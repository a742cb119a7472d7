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
// so, solving (I + L) [W | Uv] = [diag(beta gamma) K | diag(beta) V]:
//   U = Uv - W S_0^T
//   O = diag(gamma) Q S_0^T + (M o Q K^T) U,   M_{t,i} = exp(g_t - g_i) (i <= t)
//   S_C = gamma_C S_0 + U^T diag(exp(g_C - g_t)) K.
// Everything but the three products with S_0 depends on the chunk's inputs
// only: chunk_prep_kernel computes W, Uv, diag(gamma) Q, the decayed keys
// and the masked score matrix for every (head, chunk) in parallel;
// chunk_scan_kernel then walks the chunks in order for a slice of state rows
// (rows of S are independent given the shared k, q, gates).  All fp32 on
// CUDA cores with register tiles: the products are small and the state must
// stay within 1e-3 of the position-by-position recurrence.
#pragma once
#include "mk_ptx.cuh"

namespace mk {
namespace ck {

constexpr int C = 64;            // positions per chunk
constexpr int PREP_THREADS = 256;
constexpr int SCAN_THREADS = 256;
constexpr int SCAN_ROWS = 16;    // state rows per scan block

// Per (head, chunk) block of the prepared operands, in floats.  Rows of the
// [C][DK] matrices are padded to DK + 4 floats and those of P to C + 4 so a
// bulk copy lands them in the scan's conflict-free shared-memory layout.
//   W, Qg, Kd [C][DK + 4]; P [C][C + 4]; UvT [DK][C] (rows of the state);
//   gammaC (+ pad to 16 bytes)
template <int DK>
struct Blk {
  static constexpr int DKP = DK + 4;
  static constexpr int CP = C + 4;
  static constexpr int W = 0;
  static constexpr int QG = C * DKP;
  static constexpr int KD = 2 * C * DKP;
  static constexpr int P = 3 * C * DKP;
  static constexpr int UVT = 3 * C * DKP + C * CP;
  static constexpr int GC = UVT + DK * C;
  static constexpr int FLOATS = GC + 4;
};

template <int DK>
constexpr size_t prep_smem() {
  // K, Q, V [C][DK + 4]; L [C][C + 4]; g, beta, beta * gamma [C]
  return size_t(3 * C * (DK + 4) + C * (C + 4) + 3 * C) * 4;
}

// One CTA per (chunk, head).  QK [nh][T][2 DK] (normalised q | k), BAK
// [nh][T] {beta, alpha, -, -}, v of position t, head h, row r at
// V[t * v_ts + h * v_hs + r].  Positions past T are identity steps
// (beta 0, alpha 1).
template <int DK>
__global__ void __launch_bounds__(PREP_THREADS, 1) chunk_prep_kernel(
    const float* __restrict__ QK, const float4* __restrict__ BAK, const float* __restrict__ V,
    size_t v_ts, size_t v_hs, int T, float* __restrict__ out) {
  static_assert(2 * DK <= PREP_THREADS, "one thread per column of [W | Uv]");
  extern __shared__ __align__(16) float sm[];
  constexpr int LD = DK + 4, LC = C + 4;
  float* Ks = sm;
  float* Qs = Ks + C * LD;
  float* Vs = Qs + C * LD;
  float* Ls = Vs + C * LD;
  float* g = Ls + C * LC;
  float* bt = g + C;
  float* bg = bt + C;
  const int c = blockIdx.x, h = blockIdx.y, nc = gridDim.x, tid = threadIdx.x;
  const int t0 = c * C, n = min(C, T - t0);
  const float* qk = QK + (size_t(h) * T + t0) * 2 * DK;
  float* blk = out + (size_t(h) * nc + c) * Blk<DK>::FLOATS;
  for (int i = tid; i < C * DK / 4; i += PREP_THREADS) {
    const int t = i / (DK / 4), d = (i % (DK / 4)) * 4;
    const bool in = t < n;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(Qs + t * LD + d) =
        in ? *reinterpret_cast<const float4*>(qk + size_t(t) * 2 * DK + d) : z;
    *reinterpret_cast<float4*>(Ks + t * LD + d) =
        in ? *reinterpret_cast<const float4*>(qk + size_t(t) * 2 * DK + DK + d) : z;
    *reinterpret_cast<float4*>(Vs + t * LD + d) =
        in ? *reinterpret_cast<const float4*>(V + size_t(t0 + t) * v_ts + size_t(h) * v_hs + d) : z;
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
  if (tid < 32) {  // inclusive prefix sums of log alpha (two values per lane)
    const float a0 = g[2 * tid], a1 = a0 + g[2 * tid + 1];
    float run = a1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, run, o);
      if (tid >= o) run += u;
    }
    const float before = run - a1;
    g[2 * tid] = a0 + before;
    g[2 * tid + 1] = run;
  }
  __syncthreads();
  const float glast = g[C - 1];
  if (tid < C) bg[tid] = bt[tid] * expf(g[tid]);
  // Qg = diag(gamma) Q and Kd = diag(exp(g_last - g_t)) K, padded rows
  for (int i = tid; i < C * DK / 4; i += PREP_THREADS) {
    const int t = i / (DK / 4), d = (i % (DK / 4)) * 4;
    const float gq = expf(g[t]), gk = expf(glast - g[t]);
    const float4 q = *reinterpret_cast<const float4*>(Qs + t * LD + d);
    const float4 k = *reinterpret_cast<const float4*>(Ks + t * LD + d);
    *reinterpret_cast<float4*>(blk + Blk<DK>::QG + t * LD + d) =
        make_float4(gq * q.x, gq * q.y, gq * q.z, gq * q.w);
    *reinterpret_cast<float4*>(blk + Blk<DK>::KD + t * LD + d) =
        make_float4(gk * k.x, gk * k.y, gk * k.z, gk * k.w);
  }
  // K K^T and Q K^T by 4 x 4 register tiles: thread (tt, ti) takes rows
  // t = 4 tt .. 4 tt + 3 and columns i = ti, ti + 16, ti + 32, ti + 48 (the
  // interleave keeps a quarter-warp's key rows in distinct banks); columns
  // above every row of the tile are skipped.
  {
    const int tt = tid / 16, ti = tid % 16;
    const int ta = tt * 4;
    const int nb = ti > ta + 3 ? 0 : min(4, (ta + 3 - ti) / 16 + 1);
    float kk[4][4], qq[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) kk[a][b] = qq[a][b] = 0.f;
#pragma unroll 2
    for (int d = 0; d < DK; d += 4) {
      float4 kt[4], ki[4], qt[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        kt[a] = *reinterpret_cast<const float4*>(Ks + (ta + a) * LD + d);
        qt[a] = *reinterpret_cast<const float4*>(Qs + (ta + a) * LD + d);
      }
#pragma unroll
      for (int b = 0; b < 4; ++b)
        ki[b] = b < nb ? *reinterpret_cast<const float4*>(Ks + (ti + 16 * b) * LD + d)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          kk[a][b] = fmaf(kt[a].x, ki[b].x, kk[a][b]);
          kk[a][b] = fmaf(kt[a].y, ki[b].y, kk[a][b]);
          kk[a][b] = fmaf(kt[a].z, ki[b].z, kk[a][b]);
          kk[a][b] = fmaf(kt[a].w, ki[b].w, kk[a][b]);
          qq[a][b] = fmaf(qt[a].x, ki[b].x, qq[a][b]);
          qq[a][b] = fmaf(qt[a].y, ki[b].y, qq[a][b]);
          qq[a][b] = fmaf(qt[a].z, ki[b].z, qq[a][b]);
          qq[a][b] = fmaf(qt[a].w, ki[b].w, qq[a][b]);
        }
    }
    // L (strictly lower) to shared memory, P (lower incl. diagonal) out
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int t = ta + a;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int i = ti + 16 * b;
        const float dec = i <= t ? expf(g[t] - g[i]) : 0.f;
        Ls[t * LC + i] = i < t ? bt[t] * dec * kk[a][b] : 0.f;
        blk[Blk<DK>::P + t * LC + i] = i <= t ? dec * qq[a][b] : 0.f;
      }
    }
  }
  __syncthreads();
  // Forward substitution (I + L) x = b for one column of [W | Uv] per
  // thread: columns c < DK take b_t = beta_t gamma_t k_t[c], the others
  // b_t = beta_t v_t[c - DK].  The column stays in registers.
  if (tid < 2 * DK) {
    const bool isw = tid < DK;
    const int col = isw ? tid : tid - DK;
    const float* src = isw ? Ks : Vs;
    float x[C];
#pragma unroll
    for (int t = 0; t < C; ++t) {
      float s0 = (isw ? bg[t] : bt[t]) * src[t * LD + col], s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int i = 0; i + 3 < t; i += 4) {
        const float4 l = *reinterpret_cast<const float4*>(Ls + t * LC + i);
        s0 = fmaf(-l.x, x[i], s0);
        s1 = fmaf(-l.y, x[i + 1], s1);
        s2 = fmaf(-l.z, x[i + 2], s2);
        s3 = fmaf(-l.w, x[i + 3], s3);
      }
#pragma unroll
      for (int i = t & ~3; i < t; ++i) s0 = fmaf(-Ls[t * LC + i], x[i], s0);
      x[t] = (s0 + s1) + (s2 + s3);
    }
    if (isw) {
#pragma unroll
      for (int t = 0; t < C; ++t) blk[Blk<DK>::W + t * LD + col] = x[t];
    } else {
#pragma unroll
      for (int t = 0; t < C; t += 4)
        *reinterpret_cast<float4*>(blk + Blk<DK>::UVT + col * C + t) =
            make_float4(x[t], x[t + 1], x[t + 2], x[t + 3]);
    }
  }
  if (tid == 0) blk[Blk<DK>::GC] = expf(glast);
}

template <int DK>
constexpr size_t scan_smem() {
  // W, Qg, Kd [C][DK + 4]; P [C][C + 4]; UvT, UT [R][C]; S [R][DK + 4];
  // 4 mbarriers
  return size_t(3 * C * (DK + 4) + C * (C + 4) + 2 * SCAN_ROWS * C + SCAN_ROWS * (DK + 4)) * 4 +
         64;
}

// One CTA per (row slice of SCAN_ROWS rows, head): the chunks in order.  S
// [nh][DK][DK] updated in place; O[t * o_ts + h * o_hs + r] receives o.
// Each chunk's operands arrive by bulk copies (TMA) on mbarriers; a buffer's
// copy for the next chunk is issued as soon as this chunk is done with it.
// A copy that does not land within the wait bound ends the kernel early
// (the state and outputs are then incomplete).
template <int DK>
__global__ void __launch_bounds__(SCAN_THREADS, 1) chunk_scan_kernel(
    float* __restrict__ S, const float* __restrict__ prep, int T, float* __restrict__ O,
    size_t o_ts, size_t o_hs) {
  griddep_launch_dependents();
  extern __shared__ __align__(16) float sm[];
  constexpr int R = SCAN_ROWS, LD = DK + 4, LC = C + 4;
  using B = Blk<DK>;
  float* Ws = sm;
  float* Qg = Ws + C * LD;
  float* Kd = Qg + C * LD;
  float* Ps = Kd + C * LD;
  float* UvT = Ps + C * LC;
  float* UT = UvT + R * C;
  float* Ss = UT + R * C;
  uint64_t* bar = reinterpret_cast<uint64_t*>(Ss + R * LD);  // W+Qg, P, Kd, UvT
  __shared__ int bad;
  const int rs = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int r0 = rs * R, nc = (T + C - 1) / C;
  float* Sg = S + (size_t(h) * DK + r0) * DK;
  const uint64_t pol = policy_evict_last();
  // issue the copies of chunk c: which = 0 (W, Qg), 1 (P), 2 (Kd), 3 (UvT slice)
  auto load = [&](int c, int which) {
    const float* b = prep + (size_t(h) * nc + c) * B::FLOATS;
    if (which == 0) {
      mbar_arrive_expect_tx(&bar[0], 2u * C * LD * 4);
      bulk_g2s(Ws, b + B::W, C * LD * 4, &bar[0], pol);
      bulk_g2s(Qg, b + B::QG, C * LD * 4, &bar[0], pol);
    } else if (which == 1) {
      mbar_arrive_expect_tx(&bar[1], C * LC * 4);
      bulk_g2s(Ps, b + B::P, C * LC * 4, &bar[1], pol);
    } else if (which == 2) {
      mbar_arrive_expect_tx(&bar[2], C * LD * 4);
      bulk_g2s(Kd, b + B::KD, C * LD * 4, &bar[2], pol);
    } else {
      mbar_arrive_expect_tx(&bar[3], R * C * 4);
      bulk_g2s(UvT, b + B::UVT + r0 * C, R * C * 4, &bar[3], pol);
    }
  };
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bar[i], 1);
    fence_barrier_init();
    bad = 0;
  }
  for (int i = tid; i < R * DK; i += SCAN_THREADS) Ss[(i / DK) * LD + (i % DK)] = Sg[i];
  __syncthreads();
  if (tid == 0)
    for (int w = 0; w < 4; ++w) load(0, w);
  // steps 1 and 2: positions t = tp, tp + 32; rows r = 2 rp, 2 rp + 1
  const int tp = tid % 32, rp = tid / 32;
  // step 3: rows S3 * sr .. S3 * sr + S3 - 1; columns 4 dq .. 4 dq + 3
  constexpr int S3 = R / (SCAN_THREADS / (DK / 4));
  const int dq = tid % (DK / 4), sr = tid / (DK / 4);
  // bounded wait on one of the four copies of chunk c (uniform verdict)
  auto wait = [&](int i, uint32_t par) {
    const uint64_t start = global_ns();
    while (!mbar_try_wait(&bar[i], par)) {
      if (global_ns() - start > 2000000000ull) {
        bad = 1;
        break;
      }
    }
  };
  for (int c = 0; c < nc; ++c) {
    const uint32_t par = c & 1;
    wait(0, par);
    wait(3, par);
    if (__syncthreads_or(bad)) return;
    // 1: U = Uv - W S^T (to UT, transposed), Oa = Qg S^T (registers)
    float oa[2][2];
    {
      float w0[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, q0[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll 4
      for (int d = 0; d < DK; d += 4) {
        float4 wv[2], qv[2], sv[2];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          wv[a] = *reinterpret_cast<const float4*>(Ws + (tp + 32 * a) * LD + d);
          qv[a] = *reinterpret_cast<const float4*>(Qg + (tp + 32 * a) * LD + d);
          sv[a] = *reinterpret_cast<const float4*>(Ss + (2 * rp + a) * LD + d);
        }
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            w0[a][b] = fmaf(wv[a].x, sv[b].x, w0[a][b]);
            w0[a][b] = fmaf(wv[a].y, sv[b].y, w0[a][b]);
            w0[a][b] = fmaf(wv[a].z, sv[b].z, w0[a][b]);
            w0[a][b] = fmaf(wv[a].w, sv[b].w, w0[a][b]);
            q0[a][b] = fmaf(qv[a].x, sv[b].x, q0[a][b]);
            q0[a][b] = fmaf(qv[a].y, sv[b].y, q0[a][b]);
            q0[a][b] = fmaf(qv[a].z, sv[b].z, q0[a][b]);
            q0[a][b] = fmaf(qv[a].w, sv[b].w, q0[a][b]);
          }
      }
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const int t = tp + 32 * a, r = 2 * rp + b;
          UT[r * C + t] = UvT[r * C + t] - w0[a][b];
          oa[a][b] = q0[a][b];
        }
    }
    __syncthreads();  // UT complete; W, Qg, UvT free
    if (tid == 0 && c + 1 < nc) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      load(c + 1, 0);
      load(c + 1, 3);
    }
    wait(1, par);
    if (__syncthreads_or(bad)) return;
    // 2: O = Oa + (M o Q K^T) U for positions inside T (P is zero above
    // the diagonal, so the sum may run to the end of t's group of four)
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int t = tp + 32 * a;
      float o0 = oa[a][0], o1 = oa[a][1];
      for (int i = 0; i <= t; i += 4) {
        const float4 pv = *reinterpret_cast<const float4*>(Ps + t * LC + i);
        const float4 ua = *reinterpret_cast<const float4*>(UT + (2 * rp) * C + i);
        const float4 ub = *reinterpret_cast<const float4*>(UT + (2 * rp + 1) * C + i);
        o0 = fmaf(pv.x, ua.x, o0); o0 = fmaf(pv.y, ua.y, o0);
        o0 = fmaf(pv.z, ua.z, o0); o0 = fmaf(pv.w, ua.w, o0);
        o1 = fmaf(pv.x, ub.x, o1); o1 = fmaf(pv.y, ub.y, o1);
        o1 = fmaf(pv.z, ub.z, o1); o1 = fmaf(pv.w, ub.w, o1);
      }
      if (c * C + t < T) {
        float* dst = O + size_t(c * C + t) * o_ts + size_t(h) * o_hs + r0 + 2 * rp;
        dst[0] = o0;
        dst[1] = o1;
      }
    }
    wait(2, par);
    if (__syncthreads_or(bad)) return;
    // 3: S <- gamma_C S + U^T Kd
    {
      const float gc = prep[(size_t(h) * nc + c) * B::FLOATS + B::GC];
      float acc[S3][4];
#pragma unroll
      for (int a = 0; a < S3; ++a) {
        const float4 s = *reinterpret_cast<const float4*>(Ss + (S3 * sr + a) * LD + 4 * dq);
        acc[a][0] = gc * s.x;
        acc[a][1] = gc * s.y;
        acc[a][2] = gc * s.z;
        acc[a][3] = gc * s.w;
      }
#pragma unroll 2
      for (int t = 0; t < C; t += 4) {
        float4 kv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          kv[e] = *reinterpret_cast<const float4*>(Kd + (t + e) * LD + 4 * dq);
#pragma unroll
        for (int a = 0; a < S3; ++a) {
          const float4 uv = *reinterpret_cast<const float4*>(UT + (S3 * sr + a) * C + t);
          const float ue[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[a][0] = fmaf(ue[e], kv[e].x, acc[a][0]);
            acc[a][1] = fmaf(ue[e], kv[e].y, acc[a][1]);
            acc[a][2] = fmaf(ue[e], kv[e].z, acc[a][2]);
            acc[a][3] = fmaf(ue[e], kv[e].w, acc[a][3]);
          }
        }
      }
      __syncthreads();  // every read of S, UT, P and Kd for this chunk is done
#pragma unroll
      for (int a = 0; a < S3; ++a)
        *reinterpret_cast<float4*>(Ss + (S3 * sr + a) * LD + 4 * dq) =
            make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
    }
    if (tid == 0 && c + 1 < nc) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      load(c + 1, 1);
      load(c + 1, 2);
    }
    __syncthreads();  // S updated
  }
  for (int i = tid; i < R * DK; i += SCAN_THREADS) Sg[i] = Ss[(i / DK) * LD + (i % DK)];
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
