// mk_verify.cuh -- the DeltaNet mixer of a verify chunk, and rollback by
// replay.
//
// A verify call (speculative decoding: the accepted token plus drafts, one
// forward pass) must leave the model able to continue after any prefix of
// its positions.  Writing the full recurrent state after every position
// (16 heads x 128 x 128 fp32 = 1 MB per DeltaNet layer and position) costs
// more memory traffic than the state itself.  Here a verify chunk writes a
// small record per position instead -- the normalised key, the value, the
// gates alpha and beta, and the raw conv inputs of the q|k|v channels -- and
// leaves the state of the chunk's first position in place.  Accepting k
// positions marks the first k records for replay; the next call that reads
// the state applies them first (S <- alpha S + beta (v - alpha S k) k^T and
// the conv history shift, the same update as the recurrence), so no state
// after a rejected position is ever written.
//
// dn_verify_kernel: grid (heads, DK / BR, layers); each CTA owns BR = 16
// state rows of one head in registers (8 warps x 2 rows, DK / 32 entries per
// lane), replays the pending records of the previous chunk before it waits
// for the in-projection (the records and state do not depend on it), writes
// the replayed state to the next state buffer when there was anything to
// replay, then runs the causal conv + SiLU, the q/k L2 norms, the gates and
// the recurrence for the chunk's T positions, and finally the gated RMSNorm
// of each head's readout: the CTAs of one head form a thread-block cluster
// and add their rows' sums of squares through distributed shared memory, so
// the output projection reads finished operands.  With T = 0 it only
// replays (over all DeltaNet layers at once: blockIdx.z is the layer).
#pragma once
#include <cooperative_groups.h>

#include "mk_model.cuh"
#include "mk_prefill.cuh"
#include "mk_ptx.cuh"

namespace mk {
namespace vf {

constexpr int WARPS = 8;
constexpr int RPW = 2;                 // state rows per warp
constexpr int BR = WARPS * RPW;        // state rows per CTA
constexpr int THREADS = WARPS * 32;

// The record of one chunk in one DeltaNet layer (position-major).
struct Log {
  float* k;     // [kMaxVerify][nh][DK] L2-normalised keys
  float* v;     // [kMaxVerify][nh][DK] values after conv + SiLU
  float2* ab;   // [kMaxVerify][nh]     {alpha, beta}
  float* u;     // [kMaxVerify][ch]     conv inputs of the q|k|v channels
};

struct DnArgs {
  // layer 0's pointers; layer z adds z times the strides below
  const float* S_in;      // [nh][DK][DK] state before the chunk (before the replay)
  float* S_out;           // replayed state, written when R > 0 (else unused)
  const float4* conv_in;  // [ch] conv history (u_-3, u_-2, u_-1, -)
  float4* conv_out;       // replayed history, written when R > 0
  Log rlog;               // records of the previous chunk; the first R are replayed
  int R;
  Log wlog;               // this chunk's records (T > 0)
  size_t s_stride, c_stride, lk_stride, lab_stride, lu_stride;
  // this chunk (T > 0; one layer per launch)
  const float* P;         // [T][ldp] in-projection outputs: q|k|v channels, z, b, a
  int ldp;
  const uint16_t* conv_w; // [ch][4] bf16 taps, oldest first
  const float* A_log;
  const float* dt_bias;
  // [T][ldo] output: RMSNorm_DK(o_t) * out_norm * SiLU(z_t) per head, with the
  // readout o_t = S_t q_t and z_t at column zcol + h * DK of P; head h at
  // column h * DK.  out_norm == nullptr: o_t itself (no cluster launch).
  float* O;
  int ldo;
  const uint16_t* out_norm;
  float eps;
  int zcol;
  int nh, ch, T;
};

template <int DK>
__global__ void __launch_bounds__(THREADS) dn_verify_kernel(const __grid_constant__ DnArgs a) {
  constexpr int EPL = DK / 32;
  __shared__ __align__(16) float sqk[kMaxVerify][2 * DK];  // conv outputs of q | k
  __shared__ float4 sg[kMaxVerify];                          // {beta, alpha, k.q, -}
  __shared__ float sv[kMaxVerify][BR];                       // conv outputs of v (own rows)
  __shared__ float so[kMaxVerify][BR];                       // readout of the own rows
  __shared__ float pss[kMaxVerify], inv[kMaxVerify];
  griddep_launch_dependents();
  const int h = blockIdx.x, z = blockIdx.z, nh = a.nh, ch = a.ch, T = a.T;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int brow0 = blockIdx.y * BR, row0 = brow0 + warp * RPW;
  const bool lead = blockIdx.y == 0;  // writes the head's shared records and q/k history
  const float* S_in = a.S_in + z * a.s_stride + size_t(h) * DK * DK;
  const float4* conv_in = a.conv_in + z * a.c_stride;
  const float* rk = a.rlog.k + z * a.lk_stride;
  const float* rv = a.rlog.v + z * a.lk_stride;
  const float2* rab = a.rlog.ab + z * a.lab_stride;
  const float* ru = a.rlog.u + z * a.lu_stride;
  // ---- state rows, with the previous chunk's accepted positions replayed ------
  float st[RPW][EPL];
#pragma unroll
  for (int r = 0; r < RPW; ++r)
#pragma unroll
    for (int e = 0; e < EPL; ++e) st[r][e] = S_in[size_t(row0 + r) * DK + lane * EPL + e];
  for (int j = 0; j < a.R; ++j) {
    float k[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) k[e] = rk[(size_t(j) * nh + h) * DK + lane * EPL + e];
    const float2 ab = rab[size_t(j) * nh + h];
    float p0 = 0.f, p1 = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      p0 = fmaf(st[0][e], k[e], p0);
      p1 = fmaf(st[1][e], k[e], p1);
    }
    p0 = warp_sum(p0);
    p1 = warp_sum(p1);
    const float u0 = ab.y * (rv[(size_t(j) * nh + h) * DK + row0] - ab.x * p0);
    const float u1 = ab.y * (rv[(size_t(j) * nh + h) * DK + row0 + 1] - ab.x * p1);
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      st[0][e] = fmaf(ab.x, st[0][e], u0 * k[e]);
      st[1][e] = fmaf(ab.x, st[1][e], u1 * k[e]);
    }
  }
  if (a.R > 0) {
    float* S_out = a.S_out + z * a.s_stride + size_t(h) * DK * DK;
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int e = 0; e < EPL; ++e) S_out[size_t(row0 + r) * DK + lane * EPL + e] = st[r][e];
  }
  // conv channels of this CTA: the head's q and k channels (all CTAs need
  // them; the lead CTA owns them) and the CTA's BR value channels
  const int nch = 2 * DK + BR;
  auto chan = [&](int i) {
    return i < DK ? h * DK + i
                  : i < 2 * DK ? nh * DK + h * DK + (i - DK) : 2 * nh * DK + h * DK + brow0 + (i - 2 * DK);
  };
  auto history = [&](int c) {
    float4 s = conv_in[c];
    for (int j = 0; j < a.R; ++j) {
      s.x = s.y;
      s.y = s.z;
      s.z = ru[size_t(j) * ch + c];
    }
    return s;
  };
  // at most two channels per thread: history (replayed) and taps
  constexpr int CPT = (2 * DK + BR + THREADS - 1) / THREADS;
  float4 hist[CPT];
  uint2 taps[CPT];
#pragma unroll
  for (int q = 0; q < CPT; ++q) {
    const int i = tid + q * THREADS;
    if (i < nch) {
      hist[q] = history(chan(i));
      // conv_w, P and the chunk's outputs are only given when T > 0
      if (T > 0) taps[q] = *reinterpret_cast<const uint2*>(a.conv_w + size_t(chan(i)) * 4);
      if (a.R > 0 && (lead || i >= 2 * DK)) (a.conv_out + z * a.c_stride)[chan(i)] = hist[q];
    }
  }
  if (T == 0) return;
  // ---- this chunk: conv + SiLU (inputs written by the in-projection) ---------
  griddep_wait();
  float* wk = a.wlog.k;  // one layer per launch: no z offset below
#pragma unroll
  for (int q = 0; q < CPT; ++q) {
    const int i = tid + q * THREADS;
    if (i < nch) {
      const int c = chan(i);
      float u[kMaxVerify];
#pragma unroll
      for (int t = 0; t < kMaxVerify; ++t) u[t] = t < T ? a.P[size_t(t) * a.ldp + c] : 0.f;
      float4 s = hist[q];
      const float w0 = bf_lo(taps[q].x), w1 = bf_hi(taps[q].x);
      const float w2 = bf_lo(taps[q].y), w3 = bf_hi(taps[q].y);
#pragma unroll
      for (int t = 0; t < kMaxVerify; ++t) {
        if (t < T) {
          const float y = siluf_(w0 * s.x + w1 * s.y + w2 * s.z + w3 * u[t]);
          if (i < 2 * DK)
            sqk[t][i] = y;
          else
            sv[t][i - 2 * DK] = y;
          if (lead || i >= 2 * DK) a.wlog.u[size_t(t) * ch + c] = u[t];
          s.x = s.y;
          s.y = s.z;
          s.z = u[t];
        }
      }
    }
  }
  __syncthreads();
  // q / ||q|| / sqrt(DK) and k / ||k||: one warp per (position, q or k)
  for (int p = warp; p < 2 * T; p += WARPS) {
    const int t = p >> 1, isk = p & 1;
    float* x = &sqk[t][isk * DK];
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) s = fmaf(x[lane + 32 * e], x[lane + 32 * e], s);
    s = warp_sum(s);
    const float inv = 1.0f / sqrtf(s + 1e-6f);
    const float sc = isk ? 1.f : 1.0f / sqrtf(float(DK));
#pragma unroll
    for (int e = 0; e < EPL; ++e) x[lane + 32 * e] = x[lane + 32 * e] * inv * sc;
  }
  __syncthreads();
  // k.q and the gates: one warp per position
  if (warp < T) {
    const int t = warp;
    float kq = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) kq = fmaf(sqk[t][lane + 32 * e], sqk[t][DK + lane + 32 * e], kq);
    kq = warp_sum(kq);
    if (lane == 0) {
      const float* prow = a.P + size_t(t) * a.ldp;
      const float b = prow[ch + nh * DK + h], aa = prow[ch + nh * DK + nh + h];
      const float beta = sigmoidf_(b);
      const float alpha = expf(-expf(a.A_log[h]) * softplusf_(aa + a.dt_bias[h]));
      sg[t] = make_float4(beta, alpha, kq, 0.f);
      if (lead) a.wlog.ab[size_t(t) * nh + h] = make_float2(alpha, beta);
    }
  }
  __syncthreads();
  // this chunk's records: keys (lead CTA) and the CTA's values
  if (lead)
    for (int i = tid; i < T * DK; i += THREADS)
      wk[(size_t(i / DK) * nh + h) * DK + (i % DK)] = sqk[i / DK][DK + (i % DK)];
  for (int i = tid; i < T * BR; i += THREADS)
    a.wlog.v[(size_t(i / BR) * nh + h) * DK + brow0 + (i % BR)] = sv[i / BR][i % BR];
  // ---- the recurrence over the chunk; the state itself is not written ---------
  for (int t = 0; t < T; ++t) {
    float q[EPL], k[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      q[e] = sqk[t][lane * EPL + e];
      k[e] = sqk[t][DK + lane * EPL + e];
    }
    const float4 g = sg[t];
    float pk0 = 0.f, pq0 = 0.f, pk1 = 0.f, pq1 = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      pk0 = fmaf(st[0][e], k[e], pk0);
      pq0 = fmaf(st[0][e], q[e], pq0);
      pk1 = fmaf(st[1][e], k[e], pk1);
      pq1 = fmaf(st[1][e], q[e], pq1);
    }
    // lanes 0-7: S0.k, 8-15: S0.q, 16-23: S1.k, 24-31: S1.q
    const float zz = reduce4(pk0, pq0, pk1, pq1, lane);
    const float sk0 = __shfl_sync(0xffffffffu, zz, 0), sk1 = __shfl_sync(0xffffffffu, zz, 16);
    const float u0 = g.x * (sv[t][warp * RPW] - g.y * sk0);
    const float u1 = g.x * (sv[t][warp * RPW + 1] - g.y * sk1);
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      st[0][e] = fmaf(g.y, st[0][e], u0 * k[e]);
      st[1][e] = fmaf(g.y, st[1][e], u1 * k[e]);
    }
    if (lane == 8) so[t][warp * RPW] = fmaf(g.y, zz, u0 * g.z);
    if (lane == 24) so[t][warp * RPW + 1] = fmaf(g.y, zz, u1 * g.z);
  }
  // ---- gated RMSNorm over the head's DK rows, held by the CTAs of the cluster --
  __syncthreads();
  if (!a.out_norm) {
    for (int i = tid; i < T * BR; i += THREADS)
      a.O[size_t(i / BR) * a.ldo + h * DK + brow0 + i % BR] = so[i / BR][i % BR];
    return;
  }
  if (tid < T) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < BR; ++r) s = fmaf(so[tid][r], so[tid][r], s);
    pss[tid] = s;
  }
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  cl.sync();  // every CTA's partial sums written
  if (tid < T) {
    float tot = 0.f;
    for (unsigned c = 0; c < cl.num_blocks(); ++c) tot += cl.map_shared_rank(pss, c)[tid];
    inv[tid] = 1.0f / sqrtf(tot / float(DK) + a.eps);
  }
  cl.sync();  // the remote reads are done before any CTA of the cluster exits
  for (int i = tid; i < T * BR; i += THREADS) {
    const int t = i / BR, r = i % BR, row = brow0 + r;
    const float z = a.P[size_t(t) * a.ldp + a.zcol + h * DK + row];
    a.O[size_t(t) * a.ldo + h * DK + row] = so[t][r] * inv[t] * bf2f(a.out_norm[row]) * siluf_(z);
  }
}


// ---------------------------------------------------------------------------
// Causal GQA attention of a chunk of T <= 8 positions over the KV cache.
//
// attn_chunk_kernel: grid (key ranges of ATT_L positions, kv heads).  One CTA
// scores all G * T query rows of its kv head (G = q heads per kv head) against
// its key range, so each K/V row is read from memory once per chunk instead
// of once per query head and position.  The rows of earlier calls are
// staged before the kernel waits for the rope kernel in front of it (which
// appends this chunk's keys and values to the cache).  Scores and the
// weighted sum run on CUDA cores from shared memory; each range leaves an
// unnormalised partial {acc[HD], m, l}, and attn_chunk_merge combines the
// ranges in a fixed order.
constexpr int ATT_L = 32;      // keys per range (two CTAs per SM over 4K keys)
constexpr int ATT_QMAX = 32;   // query rows per kv head (G * T)
constexpr int ATT_THREADS = 256;

// QT: the query rows G * T rounded up to a multiple of 8 (one instantiation
// each, so the loops carry no idle rows beyond the last group of 8)
template <int HD, int QT>
constexpr size_t att_smem() {
  return size_t(ATT_L) * (HD + 8) * 2 + size_t(ATT_L) * HD * 2 + size_t(QT) * HD * 4 +
         size_t(QT) * ATT_L * 4;
}

struct AttArgs {
  const float* P;          // [T][ldp]: rotated q of head h at column h * HD
  int ldp;
  const uint16_t* kc;      // [nkv][max_ctx][HD] bf16 (this layer; positions < pos0 + T written)
  const uint16_t* vc;
  int max_ctx, nq, nkv, pos0, T, nsplit;
  float* part;             // [nkv][nsplit][G * T][HD + 2]
  float* out;              // merge: [T][ldo] fp32, head h at column h * HD
  int ldo;
};

template <int HD, int QT>
__global__ void __launch_bounds__(ATT_THREADS, 2) attn_chunk_kernel(const __grid_constant__ AttArgs a) {
  extern __shared__ __align__(16) unsigned char att_sm[];
  constexpr int KLD = HD + 8;  // padded key row: conflict-free 16-byte row reads
  uint16_t* Ks = reinterpret_cast<uint16_t*>(att_sm);     // [L][KLD]
  uint16_t* Vs = Ks + ATT_L * KLD;                        // [L][HD]
  float* Qs = reinterpret_cast<float*>(Vs + ATT_L * HD);  // [QT][HD], scaled by HD^-1/2
  float* Ps = Qs + QT * HD;                               // [QT][L] scores, then weights
  __shared__ float ms[QT], ls[QT];
  griddep_launch_dependents();
  const int s = blockIdx.x, g = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.nq / a.nkv, Q = G * a.T;
  const int k0 = s * ATT_L, k1 = min(k0 + ATT_L, a.pos0 + a.T), kold = min(k1, a.pos0);
  const uint16_t* K = a.kc + size_t(g) * a.max_ctx * HD;
  const uint16_t* V = a.vc + size_t(g) * a.max_ctx * HD;
  constexpr int VPR = HD / 8;  // 16-byte vectors per row
  auto stage_rows = [&](int j0, int j1) {  // asynchronous, all in flight at once
    for (int i = tid; i < (j1 - j0) * VPR; i += ATT_THREADS) {
      const int j = j0 + i / VPR, c = i % VPR;
      cp_async16(Ks + (j - k0) * KLD + c * 8, K + size_t(j) * HD + c * 8);
      cp_async16(Vs + (j - k0) * HD + c * 8, V + size_t(j) * HD + c * 8);
    }
  };
  stage_rows(k0, max(k0, kold));  // written by earlier calls
  griddep_wait();
  if (kold < k1) stage_rows(max(k0, kold), k1);  // this chunk's keys
  const float scale = 1.0f / sqrtf(float(HD));
  for (int i = tid; i < Q * (HD / 4); i += ATT_THREADS) {
    const int r = i / (HD / 4), c = i % (HD / 4);
    const int t = r / G, gi = r - t * G;
    float4 q = *reinterpret_cast<const float4*>(a.P + size_t(t) * a.ldp + (g * G + gi) * HD + c * 4);
    q.x *= scale;
    q.y *= scale;
    q.z *= scale;
    q.w *= scale;
    *reinterpret_cast<float4*>(Qs + r * HD + c * 4) = q;
  }
  cp_async_wait_all();
  __syncthreads();
  // ---- scores: thread (key j, query group qg), queries qg + SQG r ---------------
  {
    constexpr int SQG = ATT_THREADS / ATT_L, SQPT = QT / SQG;
    const int j = tid % ATT_L, qg = tid / ATT_L, kp = k0 + j;
    float sa[SQPT], sb[SQPT];  // even / odd dimensions (packed FMAs)
#pragma unroll
    for (int r = 0; r < SQPT; ++r) sa[r] = sb[r] = 0.f;
    const uint16_t* kr = Ks + j * KLD;
    for (int d = 0; d < HD; d += 8) {
      const uint4 u = *reinterpret_cast<const uint4*>(kr + d);
      const float kf[8] = {bf_lo(u.x), bf_hi(u.x), bf_lo(u.y), bf_hi(u.y),
                           bf_lo(u.z), bf_hi(u.z), bf_lo(u.w), bf_hi(u.w)};
#pragma unroll
      for (int r = 0; r < SQPT; ++r) {
        const int qi = qg + SQG * r;
        if (qi < Q) {
          const float4 q0 = *reinterpret_cast<const float4*>(Qs + qi * HD + d);
          const float4 q1 = *reinterpret_cast<const float4*>(Qs + qi * HD + d + 4);
          ffma2(sa[r], sb[r], q0.x, q0.y, kf[0], kf[1]);
          ffma2(sa[r], sb[r], q0.z, q0.w, kf[2], kf[3]);
          ffma2(sa[r], sb[r], q1.x, q1.y, kf[4], kf[5]);
          ffma2(sa[r], sb[r], q1.z, q1.w, kf[6], kf[7]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < SQPT; ++r) {
      const int qi = qg + SQG * r;
      if (qi < Q) {
        const int t = qi / G;  // causal: key position <= the query's position
        Ps[qi * ATT_L + j] = (kp < k1 && kp <= a.pos0 + t) ? sa[r] + sb[r] : -INFINITY;
      }
    }
  }
  __syncthreads();
  // ---- softmax of the range: one warp per query row ---------------------------
  for (int qi = warp; qi < Q; qi += ATT_THREADS / 32) {
    float v[ATT_L / 32];
    float m = -INFINITY;
#pragma unroll
    for (int e = 0; e < ATT_L / 32; ++e) {
      v[e] = Ps[qi * ATT_L + lane + 32 * e];
      m = fmaxf(m, v[e]);
    }
    m = warp_max(m);
    float l = 0.f;
#pragma unroll
    for (int e = 0; e < ATT_L / 32; ++e) {
      const float p = m == -INFINITY ? 0.f : expf(v[e] - m);
      Ps[qi * ATT_L + lane + 32 * e] = p;
      l += p;
    }
    l = warp_sum(l);
    if (lane == 0) {
      ms[qi] = m;
      ls[qi] = l;
    }
  }
  __syncthreads();
  // ---- weighted values: thread (4 dims, query group), queries qg + PQG r -------
  {
    constexpr int DG = HD / 4, PQG = ATT_THREADS / DG, PQPT = (QT + PQG - 1) / PQG;
    const int dg = tid % DG, qg = tid / DG, nk = k1 - k0;
    float acc[PQPT][4];
#pragma unroll
    for (int r = 0; r < PQPT; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;
    for (int j = 0; j < nk; ++j) {
      const uint2 u = *reinterpret_cast<const uint2*>(Vs + j * HD + dg * 4);
      const float v0 = bf_lo(u.x), v1 = bf_hi(u.x), v2 = bf_lo(u.y), v3 = bf_hi(u.y);
#pragma unroll
      for (int r = 0; r < PQPT; ++r) {
        const int qi = qg + PQG * r;
        if (qi < Q) {
          const float p = Ps[qi * ATT_L + j];
          ffma2(acc[r][0], acc[r][1], p, p, v0, v1);
          ffma2(acc[r][2], acc[r][3], p, p, v2, v3);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < PQPT; ++r) {
      const int qi = qg + PQG * r;
      if (qi < Q) {
        float* o = a.part + ((size_t(g) * a.nsplit + s) * Q + qi) * (HD + 2);
        o[dg * 4 + 0] = acc[r][0];
        o[dg * 4 + 1] = acc[r][1];
        o[dg * 4 + 2] = acc[r][2];
        o[dg * 4 + 3] = acc[r][3];
        if (dg == 0) {
          o[HD] = ms[qi];      // -inf when the range holds no key of this query
          o[HD + 1] = ls[qi];
        }
      }
    }
  }
}

// out[t][h] = sum_s e^(m_s - M) acc_s / sum_s e^(m_s - M) l_s over the key
// ranges.  grid (nq, T); each warp folds ranges warp, warp + 8, ... in order,
// then the eight warps are combined in order.
template <int HD>
__global__ void __launch_bounds__(ATT_THREADS) attn_chunk_merge(const __grid_constant__ AttArgs a) {
  constexpr int EPL = HD / 32, NW = ATT_THREADS / 32;
  __shared__ float wacc[NW][HD];
  __shared__ float wm[NW], wl[NW];
  griddep_launch_dependents();
  griddep_wait();
  const int h = blockIdx.x, t = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.nq / a.nkv, Q = G * a.T, g = h / G, r = t * G + (h - g * G);
  float M = -INFINITY, Lsum = 0.f, acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  constexpr int B = 4;  // ranges whose loads are in flight together
  for (int s0 = warp; s0 < a.nsplit; s0 += NW * B) {
    float mv[B], lv[B], av[B][EPL];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int s = s0 + NW * b;
      if (s < a.nsplit) {
        const float* ps = a.part + ((size_t(g) * a.nsplit + s) * Q + r) * (HD + 2);
        mv[b] = ps[HD];
        lv[b] = ps[HD + 1];
#pragma unroll
        for (int e = 0; e < EPL; ++e) av[b][e] = ps[lane * EPL + e];
      } else {
        mv[b] = -INFINITY;
        lv[b] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) av[b][e] = 0.f;
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
      if (lv[b] > 0.f) {
        const float mn = fmaxf(M, mv[b]);
        const float co = expf(M - mn), cn = expf(mv[b] - mn);
        Lsum = Lsum * co + lv[b] * cn;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = acc[e] * co + av[b][e] * cn;
        M = mn;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) wacc[warp][lane * EPL + e] = acc[e];
  if (lane == 0) {
    wm[warp] = M;
    wl[warp] = Lsum;
  }
  __syncthreads();
  for (int d = threadIdx.x; d < HD; d += ATT_THREADS) {
    float Mx = -INFINITY;
    for (int w = 0; w < NW; ++w)
      if (wl[w] > 0.f) Mx = fmaxf(Mx, wm[w]);
    float num = 0.f, den = 0.f;
    for (int w = 0; w < NW; ++w)
      if (wl[w] > 0.f) {
        const float c = expf(wm[w] - Mx);
        num = fmaf(c, wacc[w][d], num);
        den = fmaf(c, wl[w], den);
      }
    a.out[size_t(t) * a.ldo + h * HD + d] = num / den;
  }
}

// ---------------------------------------------------------------------------
// Causal GQA attention of a prompt chunk, flash style: one CTA per (block of
// 8 positions, kv head) holds the block's G x 8 query rows and walks the key
// positions 0 .. its last position in tiles of 32 (K and V double-buffered
// with cp.async), keeping a running max, sum and weighted value sum per row
// (online softmax), so no partials leave the CTA.  Scores and the weighted
// sum use the chunk kernel's thread layout and packed FMAs.  The output
// rows go out as split bf16 operands (hi, lo) of the output projection GEMM.
constexpr int PR_POS = 8;  // positions per CTA (x G query rows <= 32)

template <int HD>
constexpr size_t prompt_att_smem() {
  return size_t(2) * ATT_L * (HD + 8) * 2 + size_t(2) * ATT_L * HD * 2 +
         size_t(ATT_QMAX) * HD * 4 + size_t(ATT_QMAX) * ATT_L * 4;
}

struct PromptAttArgs {
  const float* P;      // [T][ldp] rotated q of head h at column h * HD
  int ldp;
  const uint16_t* kc;  // [nkv][max_ctx][HD] bf16, positions < pos0 + T written
  const uint16_t* vc;
  int max_ctx, nq, nkv, pos0, T;
  uint16_t* Ob;        // [T][ldo] bf16 hi (+ lo at offset lo), head h at column h * HD
  int ldo;
  size_t lo;
};

template <int HD>
__global__ void __launch_bounds__(ATT_THREADS, 2) attn_prompt_kernel(
    const __grid_constant__ PromptAttArgs a) {
  extern __shared__ __align__(16) unsigned char pa_sm[];
  constexpr int KLD = HD + 8, L = ATT_L;
  uint16_t* Ks = reinterpret_cast<uint16_t*>(pa_sm);       // [2][L][KLD]
  uint16_t* Vs = Ks + 2 * L * KLD;                         // [2][L][HD]
  float* Qs = reinterpret_cast<float*>(Vs + 2 * L * HD);   // [32][HD], scaled by HD^-1/2
  float* Ps = Qs + ATT_QMAX * HD;                          // [32][L]
  __shared__ float mrow[ATT_QMAX], lrow[ATT_QMAX], crow[ATT_QMAX];
  const int b = blockIdx.x, g = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.nq / a.nkv;
  const int t0 = b * PR_POS, tb = min(PR_POS, a.T - t0), R = tb * G;
  const int kend = a.pos0 + t0 + tb;  // keys 0 .. kend - 1 (the block's last position)
  const int ntile = (kend + L - 1) / L;
  const uint16_t* K = a.kc + size_t(g) * a.max_ctx * HD;
  const uint16_t* V = a.vc + size_t(g) * a.max_ctx * HD;
  constexpr int VPR = HD / 8;
  auto stage = [&](int tile) {
    const int j0 = tile * L, j1 = min(j0 + L, kend), buf = tile & 1;
    for (int i = tid; i < (j1 - j0) * VPR; i += ATT_THREADS) {
      const int j = i / VPR, c = i % VPR;
      cp_async16(Ks + (buf * L + j) * KLD + c * 8, K + size_t(j0 + j) * HD + c * 8);
      cp_async16(Vs + (buf * L + j) * HD + c * 8, V + size_t(j0 + j) * HD + c * 8);
    }
  };
  stage(0);
  cp_async_commit();
  const float scale = 1.0f / sqrtf(float(HD));
  for (int i = tid; i < R * (HD / 4); i += ATT_THREADS) {
    const int r = i / (HD / 4), c = i % (HD / 4);
    const int t = r / G, gi = r - t * G;
    float4 q = *reinterpret_cast<const float4*>(a.P + size_t(t0 + t) * a.ldp + (g * G + gi) * HD +
                                                c * 4);
    q.x *= scale;
    q.y *= scale;
    q.z *= scale;
    q.w *= scale;
    *reinterpret_cast<float4*>(Qs + r * HD + c * 4) = q;
  }
  if (tid < ATT_QMAX) {
    mrow[tid] = -INFINITY;
    lrow[tid] = 0.f;
  }
  constexpr int DG = HD / 4, PQG = ATT_THREADS / DG, PQPT = (ATT_QMAX + PQG - 1) / PQG;
  const int dg = tid % DG, pqg = tid / DG;
  float acc[PQPT][4];
#pragma unroll
  for (int r = 0; r < PQPT; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;
  constexpr int SQG = ATT_THREADS / L, SQPT = ATT_QMAX / SQG;
  const int j = tid % L, sqg = tid / L;
  for (int tile = 0; tile < ntile; ++tile) {
    if (tile + 1 < ntile) stage(tile + 1);
    cp_async_commit();
    cp_async_wait_all_but_one();  // this tile's keys and values have landed
    __syncthreads();
    const int buf = tile & 1, k0 = tile * L, nk = min(L, kend - k0);
    // scores of the tile, masked by position
    {
      float sa[SQPT], sb[SQPT];
#pragma unroll
      for (int r = 0; r < SQPT; ++r) sa[r] = sb[r] = 0.f;
      const uint16_t* kr = Ks + (buf * L + j) * KLD;
      for (int d = 0; d < HD; d += 8) {
        const uint4 u = *reinterpret_cast<const uint4*>(kr + d);
        const float kf[8] = {bf_lo(u.x), bf_hi(u.x), bf_lo(u.y), bf_hi(u.y),
                             bf_lo(u.z), bf_hi(u.z), bf_lo(u.w), bf_hi(u.w)};
#pragma unroll
        for (int r = 0; r < SQPT; ++r) {
          const int qi = sqg + SQG * r;
          if (qi < R) {
            const float4 q0 = *reinterpret_cast<const float4*>(Qs + qi * HD + d);
            const float4 q1 = *reinterpret_cast<const float4*>(Qs + qi * HD + d + 4);
            ffma2(sa[r], sb[r], q0.x, q0.y, kf[0], kf[1]);
            ffma2(sa[r], sb[r], q0.z, q0.w, kf[2], kf[3]);
            ffma2(sa[r], sb[r], q1.x, q1.y, kf[4], kf[5]);
            ffma2(sa[r], sb[r], q1.z, q1.w, kf[6], kf[7]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < SQPT; ++r) {
        const int qi = sqg + SQG * r;
        if (qi < R) {
          const int kp = k0 + j, qpos = a.pos0 + t0 + qi / G;
          Ps[qi * L + j] = (j < nk && kp <= qpos) ? sa[r] + sb[r] : -INFINITY;
        }
      }
    }
    __syncthreads();
    // online softmax: one warp per row, one key per lane (L == 32)
    for (int qi = warp; qi < R; qi += ATT_THREADS / 32) {
      const float s = Ps[qi * L + lane];
      const float mo = mrow[qi], mn = fmaxf(mo, warp_max(s));
      const float p = mn == -INFINITY ? 0.f : expf(s - mn);
      const float c = mo == -INFINITY ? 0.f : expf(mo - mn);
      const float ps = warp_sum(p);
      Ps[qi * L + lane] = p;
      if (lane == 0) {
        mrow[qi] = mn;
        lrow[qi] = lrow[qi] * c + ps;
        crow[qi] = c;
      }
    }
    __syncthreads();
    // weighted values: rescale the running sums, add the tile
#pragma unroll
    for (int r = 0; r < PQPT; ++r) {
      const int qi = pqg + PQG * r;
      if (qi < R) {
        const float c = crow[qi];
        acc[r][0] *= c;
        acc[r][1] *= c;
        acc[r][2] *= c;
        acc[r][3] *= c;
      }
    }
    for (int jj = 0; jj < nk; ++jj) {
      const uint2 u = *reinterpret_cast<const uint2*>(Vs + (buf * L + jj) * HD + dg * 4);
      const float v0 = bf_lo(u.x), v1 = bf_hi(u.x), v2 = bf_lo(u.y), v3 = bf_hi(u.y);
#pragma unroll
      for (int r = 0; r < PQPT; ++r) {
        const int qi = pqg + PQG * r;
        if (qi < R) {
          const float p = Ps[qi * L + jj];
          ffma2(acc[r][0], acc[r][1], p, p, v0, v1);
          ffma2(acc[r][2], acc[r][3], p, p, v2, v3);
        }
      }
    }
    __syncthreads();  // the buffers and Ps are reused by the next tile
  }
#pragma unroll
  for (int r = 0; r < PQPT; ++r) {
    const int qi = pqg + PQG * r;
    if (qi < R) {
      const float inv = 1.0f / lrow[qi];
      const int t = qi / G, h = g * G + (qi - (qi / G) * G);
      uint16_t* o = a.Ob + size_t(t0 + t) * a.ldo + h * HD + dg * 4;
      pf::store_split(o + 0, a.lo, acc[r][0] * inv);
      pf::store_split(o + 1, a.lo, acc[r][1] * inv);
      pf::store_split(o + 2, a.lo, acc[r][2] * inv);
      pf::store_split(o + 3, a.lo, acc[r][3] * inv);
    }
  }
}

}  // namespace vf
}  // namespace mk
