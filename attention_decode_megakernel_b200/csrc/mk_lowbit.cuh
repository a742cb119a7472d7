// mk_lowbit.cuh -- 4-bit weights with fp32 activations and accumulation.
//
// The tag page "RTX 3090" (the item on a custom engine for a 27B-class
// model on one RTX 3090) credits 4-bit weights with 16-bit activations
// ("W4A16") for much of its speed: a batch-1 decoder streams every weight
// once per token, so bytes per weight set the token rate.  Format here:
//   * groups of G = 64 consecutive weights of a row share one fp32 scale
//     s = max|w| / 7 (0 for an all-zero group);
//   * each weight becomes q = clamp(rint(w / s), -7, 7) (IEEE fp32 division,
//     round half to even), stored as the nibble q + 8; element k of a row
//     sits in byte k / 2, the even element in the low nibble;
//   * a row of K weights takes K / 2 bytes of codes and K / 16 bytes of
//     scales: 0.5625 bytes per weight instead of 2 for bf16.
// gemv_w4_kernel<T> computes y[t][n] = sum_k s(n, k / 64) q(n, k) x[t][k] for
// T <= 8 activation rows, every code row streamed once for all T: a CTA
// takes blocks of RW rows per warp group, kw warps split each row's K range,
// and a lane takes 16 codes at a time (8 bytes, all in one scale group).
// Decoding costs one byte permute per weight: the even and odd nibbles of a
// code word are masked into separate words, a permute places one of them in
// the mantissa of 2^23 (the float 2^23 + nibble), and one packed add of
// -(2^23 + 8) per two weights leaves q exactly.  The 16 products with each
// activation row are summed with packed fp32 FMAs and scaled by the group's
// s once.  The activation rows sit in shared memory with the four 16-byte
// pieces of every 16-weight vector in separate planes, so a warp's reads
// are consecutive 16-byte words.
#pragma once
#include "mk_ptx.cuh"

namespace mk {
namespace q4 {

constexpr int G = 64;            // weights per scale group
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int TMAX = 8;
constexpr int MAX_CTAS = 296;

constexpr int rw_for(int T) { return T <= 3 ? 4 : T <= 6 ? 2 : 1; }  // rows per warp pass (no spills)

// One thread per (row, group): scale and 32 bytes of codes.
__global__ void quantize_w4_kernel(const uint16_t* __restrict__ W, int rows, int cols,
                                   uint8_t* __restrict__ codes, float* __restrict__ scales) {
  const int gpr = cols / G;
  const size_t gid = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= size_t(rows) * gpr) return;
  const size_t row = gid / gpr;
  const int g = int(gid - row * gpr);
  const uint16_t* w = W + row * cols + size_t(g) * G;
  float amax = 0.f;
  for (int k = 0; k < G; ++k) amax = fmaxf(amax, fabsf(bf2f(w[k])));
  const float s = __fdiv_rn(amax, 7.0f);
  scales[gid] = s;
  uint8_t* c = codes + row * (cols / 2) + size_t(g) * (G / 2);
  for (int k = 0; k < G; k += 2) {
    int q0 = 0, q1 = 0;
    if (s > 0.f) {
      q0 = max(-7, min(7, int(rintf(__fdiv_rn(bf2f(w[k]), s)))));
      q1 = max(-7, min(7, int(rintf(__fdiv_rn(bf2f(w[k + 1]), s)))));
    }
    c[k / 2] = uint8_t((q0 + 8) | ((q1 + 8) << 4));
  }
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// {a, b} += {c, c}: one packed fp32 add
__device__ __forceinline__ void fadd2c(float& a, float& b, float c) {
  asm("{\n\t.reg .b64 p, q;\n\t"
      "mov.b64 p, {%0, %1};\n\t"
      "mov.b64 q, {%2, %2};\n\t"
      "add.rn.f32x2 p, p, q;\n\t"
      "mov.b64 {%0, %1}, p;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(c));
}

// Weights 2i and 2i + 1 (i < 4) of the code word w as exact floats q.
// lo / hi hold the even / odd nibbles of w, one per byte.
__device__ __forceinline__ void decode_pair(uint32_t lo, uint32_t hi, int i, float& e, float& o) {
  const uint32_t sel = uint32_t(i) | (4u << 4) | (4u << 8) | (7u << 12);  // {byte i, 0, 0, 0x4B}
  e = __uint_as_float(prmt(lo, 0x4B000000u, sel));
  o = __uint_as_float(prmt(hi, 0x4B000000u, sel));
  fadd2c(e, o, -8388616.0f);  // - (2^23 + 8)
}

template <int T>
__global__ void __launch_bounds__(THREADS, 2) gemv_w4_kernel(
    const uint8_t* __restrict__ codes, const float* __restrict__ scales,
    const float* __restrict__ x, int rows, int cols, float* __restrict__ y, int kw) {
  constexpr int RW = rw_for(T);
  extern __shared__ __align__(16) float xs[];  // [T][4 planes][cols / 16] float4
  __shared__ float red[2][WARPS][32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nv = cols / 16;  // 8-byte code vectors (16 weights) per row
  float4* x4 = reinterpret_cast<float4*>(xs);
  for (int i = tid; i < T * cols / 4; i += THREADS) {
    const int t = i / (cols / 4), f = i - t * (cols / 4);  // f: float4 index in the row
    x4[t * (cols / 4) + (f & 3) * nv + (f >> 2)] = reinterpret_cast<const float4*>(x)[i];
  }
  __syncthreads();
  const int rg = WARPS / kw, grp = warp / kw, kp = warp - grp * kw;
  const int v0 = kp * nv / kw, v1 = (kp + 1) * nv / kw;
  const int rpb = rg * RW, nblk = (rows + rpb - 1) / rpb;
  const size_t cstride = size_t(cols) / 2, sstride = size_t(cols) / G;
  int par = 0;
  for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x, par ^= 1) {
    const uint2* cr[RW];
    const float* sr[RW];
#pragma unroll
    for (int q = 0; q < RW; ++q) {
      const int n = min(blk * rpb + grp * RW + q, rows - 1);  // rows past the end repeat the last
      cr[q] = reinterpret_cast<const uint2*>(codes + size_t(n) * cstride);
      sr[q] = scales + size_t(n) * sstride;
    }
    float acc[RW][T];
#pragma unroll
    for (int q = 0; q < RW; ++q)
#pragma unroll
      for (int t = 0; t < T; ++t) acc[q][t] = 0.f;
    // one 16-weight vector of each of the RW rows: codes u, group scales s
    auto vec = [&](int v, const uint2 (&u)[RW], const float (&s)[RW]) {
      float p0[RW][T], p1[RW][T];  // the vector's even / odd products
#pragma unroll
      for (int q = 0; q < RW; ++q)
#pragma unroll
        for (int t = 0; t < T; ++t) p0[q][t] = p1[q][t] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // 4 weights (half a code word) at a time
        float xv[T][4];
#pragma unroll
        for (int t = 0; t < T; ++t) {
          const float4 p = x4[t * (cols / 4) + c * nv + v];
          xv[t][0] = p.x;
          xv[t][1] = p.y;
          xv[t][2] = p.z;
          xv[t][3] = p.w;
        }
#pragma unroll
        for (int q = 0; q < RW; ++q) {
          const uint32_t w = c < 2 ? u[q].x : u[q].y;
          const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
          float f0, f1, f2, f3;
          decode_pair(lo, hi, (c & 1) * 2, f0, f1);
          decode_pair(lo, hi, (c & 1) * 2 + 1, f2, f3);
#pragma unroll
          for (int t = 0; t < T; ++t) {
            ffma2(p0[q][t], p1[q][t], f0, f1, xv[t][0], xv[t][1]);
            ffma2(p0[q][t], p1[q][t], f2, f3, xv[t][2], xv[t][3]);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < RW; ++q)
#pragma unroll
        for (int t = 0; t < T; ++t) acc[q][t] = fmaf(s[q], p0[q][t] + p1[q][t], acc[q][t]);
    };
    for (int v = v0 + lane; v < v1; v += 64) {
      // two vectors of every row in flight per lane
      const bool two = v + 32 < v1;
      uint2 ua[RW], ub[RW];
      float sa[RW], sb[RW];
#pragma unroll
      for (int q = 0; q < RW; ++q) {
        ua[q] = __ldcs(cr[q] + v);
        sa[q] = __ldg(sr[q] + (v >> 2));  // 4 vectors per group
        if (two) {
          ub[q] = __ldcs(cr[q] + v + 32);
          sb[q] = __ldg(sr[q] + ((v + 32) >> 2));
        }
      }
      vec(v, ua, sa);
      if (two) vec(v + 32, ub, sb);
    }
    // butterfly: lane j ends with the warp's sum of value j = q * TMAX + t
    float val[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int q = i / TMAX, t = i % TMAX;
      val[i] = (q < RW && t < T) ? acc[q < RW ? q : 0][t < T ? t : 0] : 0.f;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const bool up = lane & o;
#pragma unroll
      for (int i = 0; i < o; ++i) {
        const float lo = val[i], hi = val[i + o];
        val[i] = (up ? hi : lo) + __shfl_xor_sync(0xffffffffu, up ? lo : hi, o);
      }
    }
    red[par][warp][lane] = val[0];
    __syncthreads();
    if (tid < rg * 32) {
      const int gg = tid >> 5, j = tid & 31, q = j / TMAX, t = j % TMAX;
      const int n = blk * rpb + gg * RW + q;
      if (q < RW && t < T && n < rows) {
        float sum = 0.f;
        for (int p = 0; p < kw; ++p) sum += red[par][gg * kw + p][j];
        y[size_t(t) * rows + n] = sum;
      }
    }
  }
}

// warps per row block: each lane takes about two code vectors of a row
inline int pick_kw(int cols) {
  const int nv = cols / 16;
  int kw = 1;
  while (kw < WARPS && nv / (kw * 2) >= 64) kw *= 2;
  return kw;
}

}  // namespace q4
}  // namespace mk
