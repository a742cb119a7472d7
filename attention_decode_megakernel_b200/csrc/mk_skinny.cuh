// mk_skinny.cuh -- projections of a verify chunk (a few tokens): every
// weight row streamed once for all tokens on CUDA cores.
//
// A verify call (the speculative-decoding shape: several draft tokens
// checked by one forward pass) multiplies each weight matrix by T <= 8
// activation rows.  A tensor-core tile wastes almost all of its 128 token
// columns on that shape and the call is bound by the weight stream, so here
// a CTA takes a block of weight rows, its warps split the K range of the
// block, each lane converts its 8-byte weight vectors (4 bf16) to fp32 once
// and multiplies them with all T activation rows staged in shared memory
// (16-byte reads at consecutive addresses across the warp: no bank
// conflicts).
//
// The chain of projections of one call is launched with programmatic
// stream serialisation: before it waits for the kernel in front of it, a
// CTA loads the weight vectors of its first row block into registers,
// starts an L2 prefetch of its second block and stages the norm gain, so the
// weight stream of one projection overlaps the tail of the one before.
// After the wait the T activation rows arrive by bulk copies and the
// operand's producer is applied in shared memory: RMSNorm of the residual
// stream or the gated RMSNorm of the DeltaNet readout.  The gate/up
// projection pairs gate row j with up row j in one warp and writes
// SiLU(gate) * up, so the MLP's down projection reads its operand as is.
//
// Each output is the sum of fixed K slices in a fixed order, so results do
// not depend on the grid size or on timing.
#pragma once
#include "mk.h"
#include "mk_ptx.cuh"

namespace mk {
namespace sk {

constexpr int TMAX = 8;         // tokens of one call
constexpr int THREADS = 256;    // 8 warps
constexpr int WARPS = THREADS / 32;
constexpr int RW = 4;           // weight rows per warp pass (RW * TMAX = 32 sums)
constexpr int MAX_CTAS = 296;   // two CTAs per SM on 148 SMs

enum Prologue { X_NORM = 0, X_COPY = 1, X_GATED = 2 };

struct Args {
  const uint16_t* W0;  // [N][K] bf16 rows (pair: the gate rows)
  const uint16_t* W1;  // pair: the up rows, [N][K]
  int N, K, T;
  int kw;              // warps splitting one row block's K range (1, 2, 4 or 8)
  int mode;            // Prologue
  int pair;            // C[t][j] = SiLU(W0[j] . x_t) * (W1[j] . x_t)
  // X_NORM: x = X[t][k] * rsqrt(mean_k X[t]^2 + eps) * gain[k]  (K % 128 == 0)
  // X_COPY: x = X[t][k]
  // X_GATED: x = O[t][c] * rsqrt(mean over c's head of O^2 + eps) *
  //          gain[c % dv] * SiLU(X2[t][c])       (O = X, z = X2)
  // rows of X and X2 start 16-byte aligned (ldx, ldx2, K multiples of 4)
  const float* X;
  int ldx;
  const float* X2;
  int ldx2;
  int dv;
  const uint16_t* gain;
  float eps;
  float* C;  // C[t][n] (+)= sum_k W[n][k] x[t][k], row stride ldc
  int ldc, accumulate;
  int* err;  // MK_ERR_TIMEOUT when the operand copy does not arrive
  long long wait_ns;
};

// dynamic shared memory: x rows, z rows (gated), gain (norm, gated)
constexpr size_t smem_bytes(int mode, int T, int K, int dv) {
  return size_t(T) * K * 4 * (mode == X_GATED ? 2 : 1) +
         (mode == X_NORM ? size_t(K) * 4 : mode == X_GATED ? size_t(dv) * 4 : 0);
}

// warps per row block: enough that each lane streams about four 8-byte
// vectors of every row, a power of two up to 8
inline int pick_kw(int K) {
  const int nv = K / 8;
  int kw = 1;
  while (kw < WARPS && nv / (kw * 2) >= 64) kw *= 2;
  return kw;
}

__device__ __forceinline__ float bfl(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bfh(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// dst (shared) and src (global) 16-byte aligned, bytes a multiple of 16
__device__ __forceinline__ void rows_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// 8-byte vectors of a row in flight per lane (fewer with more tokens: the
// accumulators take the registers)
constexpr int vl_for(int T) { return T <= 5 ? 4 : 2; }

// {a0, a1}[q][t] += the even / odd products of one 8-byte vector of row q with
// x_t, two at a time (packed fp32 FMA)
template <int T>
__device__ __forceinline__ void fma_vec(float (&a0)[RW][T], float (&a1)[RW][T],
                                        const uint2 (&u)[RW], const float* xs, int K, int v) {
  float w[RW][4];
#pragma unroll
  for (int q = 0; q < RW; ++q) {
    w[q][0] = bfl(u[q].x); w[q][1] = bfh(u[q].x);
    w[q][2] = bfl(u[q].y); w[q][3] = bfh(u[q].y);
  }
#pragma unroll
  for (int t = 0; t < T; ++t) {
    const float4 p = reinterpret_cast<const float4*>(xs + t * K)[v];
#pragma unroll
    for (int q = 0; q < RW; ++q) {
      ffma2(a0[q][t], a1[q][t], w[q][0], w[q][1], p.x, p.y);
      ffma2(a0[q][t], a1[q][t], w[q][2], w[q][3], p.z, p.w);
    }
  }
}

// T == a.T: one instantiation per token count, so only live accumulators
// take registers.
template <int T>
__global__ void __launch_bounds__(THREADS, 2) skinny_gemv_kernel(const __grid_constant__ Args a) {
  constexpr int VL = vl_for(T);
  extern __shared__ __align__(16) float xs[];  // [T][K] x rows, then z rows, then gain
  __shared__ float red[2][WARPS][32];
  __shared__ float inv_s[TMAX];
  __shared__ float ssp[TMAX][32];  // X_NORM: sums of squares of 128-element pieces
  __shared__ __align__(8) uint64_t bar;
  __shared__ int bad;
  griddep_launch_dependents();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K;
  const bool gated = a.mode == X_GATED;
  float* zs = xs + T * K;
  float* gs = xs + T * K * (gated ? 2 : 1);
  // ---- row blocks: rg groups of RW rows, each group's K split over kw warps --
  const int kw = a.kw, rg = WARPS / kw, g = warp / kw, kp = warp - g * kw;
  const int nv = K / 4;                       // 8-byte weight vectors per row
  const int v0 = kp * nv / kw, v1 = (kp + 1) * nv / kw;
  const int rpb = rg * RW;                    // weight rows per block
  const int lpb = a.pair ? rpb / 2 : rpb;     // output rows per block
  const int nblk = (a.N + lpb - 1) / lpb;
  auto row_ptr = [&](int blk, int q) {
    const uint16_t* w;
    if (a.pair) {
      const int j = min(blk * lpb + g * (RW / 2) + (q >> 1), a.N - 1);
      w = (q & 1 ? a.W1 : a.W0) + size_t(j) * K;
    } else {
      const int n = min(blk * rpb + g * RW + q, a.N - 1);  // rows past N repeat the last
      w = a.W0 + size_t(n) * K;
    }
    return reinterpret_cast<const uint2*>(w);
  };
  auto prefetch_blk = [&](int blk) {
    if (blk >= nblk) return;
    const int r0 = blk * lpb, nr = min(lpb, a.N - r0);
    bulk_prefetch_l2(a.W0 + size_t(r0) * K, uint32_t(nr) * K * 2);
    if (a.pair) bulk_prefetch_l2(a.W1 + size_t(r0) * K, uint32_t(nr) * K * 2);
  };
  // ---- independent of the kernel before: barrier, gain, first weights ------
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    bad = 0;
    prefetch_blk(blockIdx.x);  // the part of the first block not held in registers
    prefetch_blk(blockIdx.x + gridDim.x);
  }
  if (a.mode == X_NORM)
    for (int k = tid; k < K; k += THREADS) gs[k] = bf2f(a.gain[k]);
  else if (gated)
    for (int i = tid; i < a.dv; i += THREADS) gs[i] = bf2f(a.gain[i]);
  uint2 u[VL][RW];
  int blk = blockIdx.x;
  if (blk < nblk) {
#pragma unroll
    for (int i = 0; i < VL; ++i)
      if (v0 + lane + 32 * i < v1) {
#pragma unroll
        for (int q = 0; q < RW; ++q) u[i][q] = __ldcs(row_ptr(blk, q) + v0 + lane + 32 * i);
      }
  }
  griddep_wait();
  __syncthreads();  // barrier initialised, gain staged
  // ---- the T activation rows, written by the kernels before ------------------
  if (tid == 0) {
    const uint32_t rb = uint32_t(K) * 4;
    mbar_arrive_expect_tx(&bar, rb * T * (gated ? 2 : 1));
    for (int t = 0; t < T; ++t) {
      rows_g2s(xs + t * K, a.X + size_t(t) * a.ldx, rb, &bar);
      if (gated) rows_g2s(zs + t * K, a.X2 + size_t(t) * a.ldx2, rb, &bar);
    }
  }
  if (!mbar_try_wait(&bar, 0)) {
    const uint64_t start = global_ns();
    while (!mbar_try_wait(&bar, 0))
      if (global_ns() - start > uint64_t(a.wait_ns)) {
        bad = 1;
        break;
      }
  }
  if (__syncthreads_or(bad)) {
    if (tid == 0) atomicCAS(a.err, 0, MK_ERR_TIMEOUT);
    // the copies may still land: give them one more bounded wait
    const uint64_t start = global_ns();
    while (!mbar_try_wait(&bar, 0) && global_ns() - start < uint64_t(a.wait_ns)) {
    }
    return;
  }
  if (a.mode == X_NORM) {
    // x * gain in place, and the sums of squares of x in 128-element pieces
    // (K a multiple of 128: a warp's 32 float4 never straddle two rows); the
    // factor rsqrt(mean x^2 + eps) multiplies the dot products at the end
    const int k4 = K / 4;
    for (int i = tid; i < T * k4; i += THREADS) {
      const int t = i / k4, kk = i - t * k4;
      float4 v = reinterpret_cast<float4*>(xs)[i];
      const float4 gk = reinterpret_cast<const float4*>(gs)[kk];
      float s = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, v.w * v.w)));
      s = warp_sum(s);
      if (lane == 0) ssp[t][kk >> 5] = s;
      v.x *= gk.x;
      v.y *= gk.y;
      v.z *= gk.z;
      v.w *= gk.w;
      reinterpret_cast<float4*>(xs)[i] = v;
    }
    __syncthreads();
    if (tid < T) {
      float tot = 0.f;
      for (int c = 0; c < (k4 >> 5); ++c) tot += ssp[tid][c];
      inv_s[tid] = 1.0f / sqrtf(tot / float(K) + a.eps);
    }
  } else if (gated) {
    // one warp per (token, head); dv a multiple of 32
    const int nh = K / a.dv, per = a.dv / 32;
    for (int p = warp; p < T * nh; p += WARPS) {
      const int t = p / nh, h = p - t * nh;
      float* o = xs + t * K + h * a.dv;
      const float* z = zs + t * K + h * a.dv;
      float s = 0.f;
      for (int e = 0; e < per; ++e) {
        const float v = o[lane + 32 * e];
        s = fmaf(v, v, s);
      }
      const float inv = 1.0f / sqrtf(warp_sum(s) / float(a.dv) + a.eps);
      for (int e = 0; e < per; ++e) {
        const int i = lane + 32 * e;
        o[i] = o[i] * inv * gs[i] * siluf_(z[i]);
      }
    }
  }
  __syncthreads();
  int par = 0;
  bool first = true;  // u already holds the first vectors
  for (; blk < nblk; blk += gridDim.x, par ^= 1) {
    if (tid == 0) prefetch_blk(blk + 2 * gridDim.x);
    const uint2* wr[RW];
#pragma unroll
    for (int q = 0; q < RW; ++q) wr[q] = row_ptr(blk, q);
    float a0[RW][T], a1[RW][T];
#pragma unroll
    for (int q = 0; q < RW; ++q)
#pragma unroll
      for (int t = 0; t < T; ++t) a0[q][t] = a1[q][t] = 0.f;
    for (int v = v0 + lane; v < v1; v += 32 * VL) {
      if (!first) {
#pragma unroll
        for (int i = 0; i < VL; ++i)
          if (v + 32 * i < v1) {
#pragma unroll
            for (int q = 0; q < RW; ++q) u[i][q] = __ldcs(wr[q] + v + 32 * i);
          }
      }
      first = false;
#pragma unroll
      for (int i = 0; i < VL; ++i)
        if (v + 32 * i < v1) fma_vec<T>(a0, a1, u[i], xs, K, v + 32 * i);
    }
    first = false;
    // butterfly: after five exchanges lane j holds the warp's sum of value
    // j = q * TMAX + t
    float val[RW * TMAX];
#pragma unroll
    for (int q = 0; q < RW; ++q)
#pragma unroll
      for (int t = 0; t < TMAX; ++t) val[q * TMAX + t] = t < T ? a0[q][t] + a1[q][t] : 0.f;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const bool up = lane & o;
#pragma unroll
      for (int i = 0; i < o; ++i) {
        const float lo = val[i], hi = val[i + o];
        const float send = up ? lo : hi;
        val[i] = (up ? hi : lo) + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    red[par][warp][lane] = val[0];
    __syncthreads();
    if (tid < rg * 32) {  // one warp per row group
      const int gg = tid >> 5, j = tid & 31, q = j / TMAX, t = j % TMAX;
      float s = 0.f;
      for (int p = 0; p < kw; ++p) s += red[par][gg * kw + p][j];
      if (a.mode == X_NORM && t < T) s *= inv_s[t];
      if (a.pair) {
        // rows q (gate) and q + 1 (up) of the same output j; q even
        const float upv = __shfl_down_sync(0xffffffffu, s, TMAX);
        const int n = blk * lpb + gg * (RW / 2) + (q >> 1);
        if (!(q & 1) && t < T && n < a.N) a.C[size_t(t) * a.ldc + n] = siluf_(s) * upv;
      } else {
        const int n = blk * rpb + gg * RW + q;
        if (t < T && n < a.N) {
          float* dst = a.C + size_t(t) * a.ldc + n;
          *dst = a.accumulate ? *dst + s : s;
        }
      }
    }
  }
}

}  // namespace sk
}  // namespace mk
