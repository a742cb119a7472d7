// mk_delta.cuh -- isolated gated delta-rule step over a batch of sequences.
//
// One launch advances B x heads recurrences by one token, in place:
//   S <- alpha S (I - beta k k^T) + beta v k^T ,  o = S q
// (Gated Delta Networks, Yang, Kautz & Hatamizadeh, ICLR 2025, the gated
// delta rule).  Row i of S only needs (S_i, k, q, v_i, alpha, beta), so each
// warp streams whole 128-float rows HBM -> registers -> HBM with 16-byte
// coalesced accesses; with Sk_i = S_i.k and Sq_i = S_i.q,
//   S_i' = alpha S_i + u k ,  u = beta (v_i - alpha Sk_i) ,
//   o_i  = S_i'.q = alpha Sq_i + u (k.q).
// HBM-bound: 2 x 4 x dk bytes of state per row and step.
#pragma once
#include "mk_ptx.cuh"

namespace mk {

constexpr int DS_ROWS = 32;      // state rows per CTA
constexpr int DS_THREADS = 256;  // 8 warps, 4 rows each

template <int D>
__global__ void __launch_bounds__(DS_THREADS) delta_step_kernel(
    float* __restrict__ S, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
    const uint16_t* __restrict__ v, const float* __restrict__ alpha,
    const float* __restrict__ beta, float* __restrict__ o) {
  constexpr int EPL = D / 32;
  constexpr int RPW = DS_ROWS / (DS_THREADS / 32);
  __shared__ float qs[D], ks[D];
  __shared__ float kq_s;
  const int bh = blockIdx.x;
  const int row0 = blockIdx.y * DS_ROWS;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < D; i += DS_THREADS) {
    qs[i] = bf2f(q[size_t(bh) * D + i]);
    ks[i] = bf2f(k[size_t(bh) * D + i]);
  }
  __syncthreads();
  if (warp == 0) {
    float s = 0.f;
    for (int i = lane; i < D; i += 32) s = fmaf(ks[i], qs[i], s);
    s = warp_sum(s);
    if (lane == 0) kq_s = s;
  }
  __syncthreads();
  const float al = alpha[bh], be = beta[bh], kq = kq_s;
  float kv[EPL], qv[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    kv[e] = ks[lane * EPL + e];
    qv[e] = qs[lane * EPL + e];
  }
  float sv[RPW][EPL];
#pragma unroll
  for (int j = 0; j < RPW; ++j) {
    const int r = row0 + warp + j * (DS_THREADS / 32);
    const float* src = S + (size_t(bh) * D + r) * D + lane * EPL;
    if constexpr (EPL == 4) {
      float4 t = __ldcs(reinterpret_cast<const float4*>(src));
      sv[j][0] = t.x; sv[j][1] = t.y; sv[j][2] = t.z; sv[j][3] = t.w;
    } else {
      float2 t = __ldcs(reinterpret_cast<const float2*>(src));
      sv[j][0] = t.x; sv[j][1] = t.y;
    }
  }
#pragma unroll
  for (int j = 0; j < RPW; ++j) {
    const int r = row0 + warp + j * (DS_THREADS / 32);
    float sk = 0.f, sq = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      sk = fmaf(sv[j][e], kv[e], sk);
      sq = fmaf(sv[j][e], qv[e], sq);
    }
    sk = warp_sum(sk);
    sq = warp_sum(sq);
    const float u = be * (bf2f(v[size_t(bh) * D + r]) - al * sk);
    float* dst = S + (size_t(bh) * D + r) * D + lane * EPL;
    if constexpr (EPL == 4) {
      __stcs(reinterpret_cast<float4*>(dst),
             make_float4(fmaf(al, sv[j][0], u * kv[0]), fmaf(al, sv[j][1], u * kv[1]),
                         fmaf(al, sv[j][2], u * kv[2]), fmaf(al, sv[j][3], u * kv[3])));
    } else {
      __stcs(reinterpret_cast<float2*>(dst),
             make_float2(fmaf(al, sv[j][0], u * kv[0]), fmaf(al, sv[j][1], u * kv[1])));
    }
    if (lane == 0) o[size_t(bh) * D + r] = fmaf(al, sq, u * kq);
  }
}

}  // namespace mk
