// mk_prefill.cuh -- the multi-token (prompt) path: the stack over T
// positions at once, with the projections as tensor-core GEMMs.
//
// The launch post ("OS Megakernel that match M5 Max Tok/w at 2x the
// Throughput on RTX 3090", results table: prefill pp520) measures prompt
// processing next to decode; the operations are the decode step's, applied
// to T positions: every projection becomes a GEMM with M = T tokens, the
// causal convolution and the gated delta rule advance position by position,
// and attention is causal over the prompt plus the cached context.
//
// B200 structure: the GEMMs run on the 5th-generation tensor cores -- TMA 2D
// tile loads (128-byte swizzle) into a 4-stage shared-memory ring, one thread
// issuing tcgen05.mma (bf16 x bf16 -> fp32, M=128 weight rows x N=128
// tokens x K=16) into a TMEM accumulator, the epilogue reading TMEM with
// tcgen05.ld.  The weights are bf16 already; an fp32 activation x enters as
// two bf16 operands, hi = bf16(x) and lo = bf16(x - hi), multiplied into the
// same accumulator, so the product carries ~16 mantissa bits of x (the
// single-operand form would round every activation to 8 bits).
#pragma once
#include <cuda.h>

#include "mk_model.cuh"
#include "mk_ptx.cuh"

namespace mk {
namespace pf {

constexpr int BM = 128;       // weight rows per tile (MMA M)
constexpr int BN = 128;       // tokens per tile (MMA N)
constexpr int BK = 64;        // K elements per stage (one 128-byte swizzle span)
constexpr int STAGES = 4;
constexpr int GEMM_THREADS = 128;
constexpr uint32_t TILE_W_BYTES = BM * BK * 2;
constexpr uint32_t TILE_X_BYTES = BN * BK * 2;
constexpr uint32_t STAGE_BYTES = TILE_W_BYTES + 2 * TILE_X_BYTES;  // W, x_hi, x_lo
constexpr size_t GEMM_SMEM = size_t(STAGES) * STAGE_BYTES + 1024 + 256;

struct GemmArgs {
  CUtensorMap tw;    // weights [n_out][K] bf16, box {BK, BM}
  CUtensorMap tx;    // activations [2][x_lo_row][K] bf16 (hi rows, then lo rows), box {BK, BN}
  float* c;          // output [T][ldc] fp32, column = weight row
  int ldc;
  int n_out, T, K;
  int x_lo_row;      // row of the lo half's first row in tx
  int k_split;       // gridDim.z: K ranges summed into c with atomic adds (c pre-set by the caller)
  int accumulate;    // 1: c += result (residual add)
  int* err;
  long long wait_ns;
};

// ---- PTX wrappers for the tensor-core path ----------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes grouped by 8 (stride 1024 bytes between 8-row groups).
__device__ __forceinline__ uint64_t smem_desc_sw128(const void* p) {
  const uint64_t addr = smem_addr(p);
  return ((addr >> 4) & 0x3FFFull)       // start address (16-byte units)
         | (1ull << 16)                  // leading byte offset (unused by this layout)
         | (64ull << 32)                 // stride byte offset: 1024 B
         | (1ull << 46)                  // descriptor version
         | (2ull << 61);                 // layout: 128-byte swizzle
}

// Instruction descriptor of kind::f16: bf16 x bf16 -> fp32, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int m, int n) {
  return (1u << 4)                       // D format: f32
         | (1u << 7)                     // A format: bf16
         | (1u << 10)                    // B format: bf16
         | (uint32_t(n >> 3) << 17)      // N / 8
         | (uint32_t(m >> 4) << 24);     // M / 16
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// 32 lanes x 16 consecutive 32-bit columns (lane = TMEM lane of this warp).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

struct GemmSmem {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc;
  uint32_t tmem_base;
  int abort_flag;
};

// Wait for an mbarrier phase, bounded; returns false on timeout.
__device__ __forceinline__ bool gemm_wait(uint64_t* bar, uint32_t parity, GemmSmem* gs,
                                          int* err, long long wait_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t start = global_ns();
  for (int it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31) == 0) {
      if (*(volatile int*)&gs->abort_flag) return false;
      if (global_ns() - start > uint64_t(wait_ns)) {
        atomicCAS(err, 0, MK_ERR_TIMEOUT);
        *(volatile int*)&gs->abort_flag = 1;
        return false;
      }
    }
  }
}

// C[t][n] (+)= sum_k X[t][k] * W[n][k] for one 128 x 128 (rows x tokens) tile.
// PARTIAL: K range blockIdx.z stores its sum to partial[z][T][n_out] (summed
// afterwards in a fixed order) instead of writing c.
template <bool PARTIAL>
__device__ __forceinline__ void gemm_tile(const GemmArgs& a, float* partial) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sW = base;
  unsigned char* sX = base + size_t(STAGES) * TILE_W_BYTES;  // [STAGES][2] x tiles
  GemmSmem* gs = reinterpret_cast<GemmSmem*>(sX + size_t(STAGES) * 2 * TILE_X_BYTES);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * BM, t0 = blockIdx.y * BN;
  // this CTA's share of the K blocks (split-K when few output tiles exist)
  const int kb_all = a.K / BK;
  const int kb0 = int(blockIdx.z) * kb_all / a.k_split;
  const int nkb = (int(blockIdx.z) + 1) * kb_all / a.k_split - kb0;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&gs->full[s], 1);
      mbar_init(&gs->empty[s], 1);
    }
    mbar_init(&gs->acc, 1);
    gs->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(&gs->tmem_base, BN);  // BN fp32 columns x 128 lanes
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = gs->tmem_base;

  if (warp == 0 && lane == 0) {
    // TMA producer
    int issued = 0;
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % STAGES;
      if (kb >= STAGES && !gemm_wait(&gs->empty[s], ((kb / STAGES) - 1) & 1, gs, a.err, a.wait_ns))
        break;
      mbar_arrive_expect_tx(&gs->full[s], STAGE_BYTES);
      unsigned char* xs = sX + size_t(s) * 2 * TILE_X_BYTES;
      const int kc = (kb0 + kb) * BK;
      tma_load_2d(sW + size_t(s) * TILE_W_BYTES, &a.tw, kc, n0, &gs->full[s]);
      tma_load_2d(xs, &a.tx, kc, t0, &gs->full[s]);
      tma_load_2d(xs + TILE_X_BYTES, &a.tx, kc, a.x_lo_row + t0, &gs->full[s]);
      ++issued;
    }
    // copies still in flight must land before the CTA can exit
    for (int kb = issued - STAGES > 0 ? issued - STAGES : 0; kb < issued; ++kb) {
      const uint64_t start = global_ns();
      while (!mbar_try_wait(&gs->full[kb % STAGES], (kb / STAGES) & 1))
        if (global_ns() - start > uint64_t(a.wait_ns)) break;
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    const uint32_t idesc = idesc_bf16_f32(BM, BN);
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % STAGES;
      if (!gemm_wait(&gs->full[s], (kb / STAGES) & 1, gs, a.err, a.wait_ns)) break;
      tc_fence_after();
      const unsigned char* w = sW + size_t(s) * TILE_W_BYTES;
      const unsigned char* x = sX + size_t(s) * 2 * TILE_X_BYTES;
#pragma unroll
      for (int k = 0; k < BK / 16; ++k) {
        const uint64_t wd = smem_desc_sw128(w + k * 32);
        tc_mma(tmem, wd, smem_desc_sw128(x + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
        tc_mma(tmem, wd, smem_desc_sw128(x + TILE_X_BYTES + k * 32), idesc, 1u);
      }
      tc_commit(&gs->empty[s]);  // frees the stage once these MMAs have read it
    }
    tc_commit(&gs->acc);  // also issued after an abort: the epilogue must not hang
  }
  __syncwarp();
  // epilogue: warp w owns TMEM lanes [32w, 32w+32) = weight rows n0 + 32w + lane
  const bool ok = gemm_wait(&gs->acc, 0, gs, a.err, a.wait_ns) && !gs->abort_flag;
  tc_fence_after();
  const int n = n0 + warp * 32 + lane;
  if (ok) {
    for (int c0 = 0; c0 < BN; c0 += 16) {
      float v[16];
      tmem_ld16(tmem + (uint32_t(warp * 32) << 16) + uint32_t(c0), v);
      if (n < a.n_out) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int t = t0 + c0 + i;
          if (t < a.T) {
            float* dst = a.c + size_t(t) * a.ldc + n;
            if constexpr (PARTIAL) partial[(size_t(blockIdx.z) * a.T + t) * a.n_out + n] = v[i];
            else if (a.k_split > 1) atomicAdd(dst, v[i]);
            else *dst = a.accumulate ? *dst + v[i] : v[i];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, BN);
}

__global__ void __launch_bounds__(GEMM_THREADS, 1) gemm_tc(const __grid_constant__ GemmArgs a) {
  gemm_tile<false>(a, nullptr);
}

__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_partial(const __grid_constant__ GemmArgs a, float* partial) {
  gemm_tile<true>(a, partial);
}

// C[t][n] = sum over z of partial[z][t][n], in order z = 0, 1, ... (a split-K
// result that does not depend on the order the ranges finished in).  When
// the GEMM's wait-error word is set (a tile gave up and left its partial
// unwritten) every element of C becomes NaN instead.
__global__ void splitk_reduce_kernel(const float* partial, int k_split, size_t n, float* c,
                                     const int* err) {
  const bool failed = err && *reinterpret_cast<const volatile int*>(err) != 0;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += size_t(gridDim.x) * blockDim.x) {
    float acc = 0.f;
    for (int z = 0; z < k_split; ++z) acc += partial[size_t(z) * n + i];
    c[i] = failed ? __int_as_float(0x7FC00000) : acc;
  }
}

// C becomes NaN when the GEMM's wait-error word is set (a tile gave up and
// left its part of C unwritten).
__global__ void poison_on_error_kernel(const int* err, size_t n, float* c) {
  if (*reinterpret_cast<const volatile int*>(err) == 0) return;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += size_t(gridDim.x) * blockDim.x)
    c[i] = __int_as_float(0x7FC00000);
}

// c[t][n] (+)= sum over z of partial[z][t][n] (z = 0, 1, ... in order), for
// a split-K GEMM whose output has row stride ldc.
__global__ void splitk_reduce_ld_kernel(const float* partial, int k_split, int T, int n_out,
                                        float* c, int ldc, int accumulate) {
  const size_t n = size_t(T) * n_out;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += size_t(gridDim.x) * blockDim.x) {
    float acc = 0.f;
    for (int z = 0; z < k_split; ++z) acc += partial[size_t(z) * n + i];
    float* dst = c + (i / n_out) * size_t(ldc) + (i % n_out);
    *dst = accumulate ? *dst + acc : acc;
  }
}

// ---- elementwise / row kernels --------------------------------------------------
constexpr int ROW_THREADS = 256;

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < int(blockDim.x >> 5); ++i) s += red[i];
  return s;
}

// The two bf16 operands of an fp32 activation: hi at p[0], lo at p[lo].
__device__ __forceinline__ void store_split(uint16_t* p, size_t lo, float v) {
  const uint16_t h = f2bf(v);
  p[0] = h;
  p[lo] = f2bf(v - bf2f(h));
}

// x[t] = embedding row of tokens[t] (fp32)
__global__ void embed_kernel(const int32_t* tokens, const uint16_t* E, float* X, int H) {
  griddep_launch_dependents();
  const int t = blockIdx.x;
  const uint16_t* row = E + size_t(tokens[t]) * H;
  for (int i = threadIdx.x; i < H; i += blockDim.x) X[size_t(t) * H + i] = bf2f(row[i]);
}

// Xn[t] = split(RMSNorm(X[t]) * gain); the lo operands `lo` elements on
__global__ void rmsnorm_bf16_kernel(const float* X, const uint16_t* gain, uint16_t* Xn, int H,
                                    float eps, size_t lo) {
  __shared__ float red[32];
  const int t = blockIdx.x;
  const float* x = X + size_t(t) * H;
  float ss = 0.f;
  for (int i = threadIdx.x; i < H; i += blockDim.x) ss = fmaf(x[i], x[i], ss);
  const float inv = 1.0f / sqrtf(block_sum(ss, red) / float(H) + eps);
  for (int i = threadIdx.x; i < H; i += blockDim.x)
    store_split(Xn + size_t(t) * H + i, lo, x[i] * inv * bf2f(gain[i]));
}

// Causal depthwise conv + SiLU over T positions, one thread per (position,
// channel): Cv[t][c] = SiLU(w0 u_{t-3} + w1 u_{t-2} + w2 u_{t-1} + w3 u_t)
// with u = the raw in-projection columns of P and u_{<0} taken from the
// carried history `state` = (u_{-3}, u_{-2}, u_{-1}).
__device__ __forceinline__ float conv_input(const float* P, int ldp, const float4& s, int t,
                                            int c) {
  return t >= 0 ? P[size_t(t) * ldp + c] : (t == -1 ? s.z : t == -2 ? s.y : s.x);
}

__global__ void conv_kernel(const float* P, int ldp, const float4* state, const uint16_t* conv_w,
                            int ch, float* Cv, int ldc) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x, t = blockIdx.y;
  if (c >= ch) return;
  const float4 s = state[c];
  const uint2 wc = *reinterpret_cast<const uint2*>(conv_w + size_t(c) * 4);
  const float u3 = conv_input(P, ldp, s, t - 3, c), u2 = conv_input(P, ldp, s, t - 2, c);
  const float u1 = conv_input(P, ldp, s, t - 1, c), u0 = P[size_t(t) * ldp + c];
  const float y = bf_lo(wc.x) * u3 + bf_hi(wc.x) * u2 + bf_lo(wc.y) * u1 + bf_hi(wc.y) * u0;
  Cv[size_t(t) * ldc + c] = siluf_(y);
}

// The carried history after T positions (a separate launch: every conv
// thread must have read the old one first).
__global__ void conv_state_kernel(const float* P, int ldp, float4* state, int ch, int T) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= ch) return;
  const float4 s = state[c];
  state[c] = make_float4(conv_input(P, ldp, s, T - 3, c), conv_input(P, ldp, s, T - 2, c),
                         conv_input(P, ldp, s, T - 1, c), 0.f);
}

// Per (position, head): L2-normalised q (scaled by dk^-1/2) and k, the gates
// beta = sigmoid(b) and alpha = exp(-exp(A_log) softplus(a + dt_bias)), and
// k.q.  QK [nh][T][2*dk], BAK [nh][T][4] = {beta, alpha, k.q, 0}.
__global__ void dn_prep_kernel(const float* Cv, int ldc, const float* P, int ldp, int nh, int dk,
                               int ch, int dv, const float* A_log, const float* dt_bias,
                               float* QK, float4* BAK, int T) {
  __shared__ float red[32];
  const int t = blockIdx.x, h = blockIdx.y, i = threadIdx.x;  // blockDim.x == dk
  const float* prow = P + size_t(t) * ldp;
  const float* crow = Cv + size_t(t) * ldc;
  const float q = crow[h * dk + i], k = crow[nh * dk + h * dk + i];
  const float sq = block_sum(q * q, red);
  const float sk = block_sum(k * k, red);
  const float qn = q / sqrtf(sq + 1e-6f) / sqrtf(float(dk));
  const float kn = k / sqrtf(sk + 1e-6f);
  const float kq = block_sum(qn * kn, red);
  float* dst = QK + (size_t(h) * T + t) * 2 * dk;
  dst[i] = qn;
  dst[dk + i] = kn;
  if (i == 0) {
    const float b = prow[ch + nh * dv + h], aa = prow[ch + nh * dv + nh + h];
    BAK[size_t(h) * T + t] =
        make_float4(sigmoidf_(b), expf(-expf(A_log[h]) * softplusf_(aa + dt_bias[h])), kq, 0.f);
  }
}

// G[t][h*dv + i] = split(RMSNorm_dv(O[t][h]) * w_i * SiLU(z[t][h*dv+i]))
__global__ void gated_norm_kernel(const float* O, int ldo, const float* P, int ldp, int zcol,
                                  const uint16_t* w, uint16_t* G, int ldg, float eps, size_t lo) {
  __shared__ float red[32];
  const int t = blockIdx.x, h = blockIdx.y, i = threadIdx.x, dv = blockDim.x;
  const float o = O[size_t(t) * ldo + h * dv + i];
  const float inv = 1.0f / sqrtf(block_sum(o * o, red) / float(dv) + eps);
  const float z = P[size_t(t) * ldp + zcol + h * dv + i];
  store_split(G + size_t(t) * ldg + h * dv + i, lo, o * inv * bf2f(w[i]) * siluf_(z));
}

// Hb[t][j] = split(SiLU(gate) * up), gate at P[t][j], up at P[t][I + j]
__global__ void swiglu_kernel(const float* P, int ldp, int I, uint16_t* Hb, int ldh, size_t lo) {
  const int t = blockIdx.y;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < I; j += gridDim.x * blockDim.x)
    store_split(Hb + size_t(t) * ldh + j, lo,
                siluf_(P[size_t(t) * ldp + j]) * P[size_t(t) * ldp + I + j]);
}

// RoPE on q (in place, fp32) and k, then K/V of positions pos0 .. pos0+T-1
// into the bf16 cache.  grid (T, nq + nkv), blockDim = hd / 2.
__global__ void rope_kv_kernel(float* P, int ldp, int nq, int nkv, int hd, uint16_t* kc,
                               uint16_t* vc, int max_ctx, int pos0, float theta) {
  griddep_launch_dependents();
  griddep_wait();
  const int t = blockIdx.x, hh = blockIdx.y, i = threadIdx.x, half = hd / 2;
  const int pos = pos0 + t;
  const double inv_freq = pow(double(theta), -2.0 * double(i) / double(hd));
  double sd, cd;
  sincos(double(pos) * inv_freq, &sd, &cd);
  const float cs = float(cd), sn = float(sd);
  float* row = P + size_t(t) * ldp;
  if (hh < nq) {
    float* q = row + hh * hd;
    const float x0 = q[i], x1 = q[i + half];
    q[i] = x0 * cs - x1 * sn;
    q[i + half] = x1 * cs + x0 * sn;
  } else {
    const int g = hh - nq;
    const float* k = row + nq * hd + g * hd;
    const float* v = row + (nq + nkv) * hd + g * hd;
    const float x0 = k[i], x1 = k[i + half];
    const size_t o = (size_t(g) * max_ctx + pos) * hd;
    kc[o + i] = f2bf(x0 * cs - x1 * sn);
    kc[o + i + half] = f2bf(x1 * cs + x0 * sn);
    vc[o + i] = f2bf(v[i]);
    vc[o + i + half] = f2bf(v[i + half]);
  }
}

// EPL consecutive bf16 values -> fp32 (one 4/8/16-byte load).
template <int EPL>
__device__ __forceinline__ void load_bf16_row(const uint16_t* p, float* f) {
  if constexpr (EPL == 8) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    f[0] = bf_lo(u.x); f[1] = bf_hi(u.x); f[2] = bf_lo(u.y); f[3] = bf_hi(u.y);
    f[4] = bf_lo(u.z); f[5] = bf_hi(u.z); f[6] = bf_lo(u.w); f[7] = bf_hi(u.w);
  } else if constexpr (EPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    f[0] = bf_lo(u.x); f[1] = bf_hi(u.x); f[2] = bf_lo(u.y); f[3] = bf_hi(u.y);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    f[0] = bf_lo(u); f[1] = bf_hi(u);
  }
}

// Causal attention of T new positions over the cache (positions 0 ..
// pos0+t for query t): one warp per (query, head), online softmax; the
// output is written as split bf16 operands for the output-projection GEMM.
template <int HD>
__global__ void attn_prefill_kernel(const float* P, int ldp, const uint16_t* kc,
                                    const uint16_t* vc, int max_ctx, int nq, int nkv, int pos0,
                                    int T, uint16_t* Ob, int ldob, size_t lo) {
  constexpr int EPL = HD / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q_idx = blockIdx.x * (blockDim.x >> 5) + warp;  // query position within the chunk
  const int h = blockIdx.y;
  if (q_idx >= T) return;
  const int g = h / (nq / nkv);
  const float* qrow = P + size_t(q_idx) * ldp + h * HD;
  float q[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) q[e] = qrow[lane * EPL + e];
  const float scale = 1.0f / sqrtf(float(HD));
  const uint16_t* K = kc + size_t(g) * max_ctx * HD;
  const uint16_t* V = vc + size_t(g) * max_ctx * HD;
  float m = -INFINITY, l = 0.f, acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  const int nkeys = pos0 + q_idx + 1;
  constexpr int KB = 4;  // keys in flight per step
  for (int j0 = 0; j0 < nkeys; j0 += KB) {
    float kf[KB][EPL], vf[KB][EPL], s[KB];
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      const int j = min(j0 + u, nkeys - 1);
      load_bf16_row<EPL>(K + size_t(j) * HD + lane * EPL, kf[u]);
      load_bf16_row<EPL>(V + size_t(j) * HD + lane * EPL, vf[u]);
    }
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      s[u] = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) s[u] = fmaf(q[e], kf[u][e], s[u]);
    }
#pragma unroll
    for (int u = 0; u < KB; ++u) s[u] = warp_sum(s[u]) * scale;
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      if (j0 + u < nkeys) {
        const float mn = fmaxf(m, s[u]);
        const float corr = expf(m - mn), p = expf(s[u] - mn);
        l = l * corr + p;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = fmaf(p, vf[u][e], acc[e] * corr);
        m = mn;
      }
    }
  }
  uint16_t* orow = Ob + size_t(q_idx) * ldob + h * HD + lane * EPL;
#pragma unroll
  for (int e = 0; e < EPL; ++e) store_split(orow + e, lo, acc[e] / l);
}

// Short chunks (verify): attention split over the keys as well, so a few
// queries over a long cache still occupy the GPU.  One warp per (query t,
// head h, key range s of ATT_SPLIT_LEN positions) writes an unnormalised
// partial {acc[HD], m, l}; attn_merge_kernel combines the ranges.
constexpr int ATT_SPLIT_LEN = 64;
constexpr int ATT_SPLIT_WARPS = 4;

template <int HD>
__global__ void __launch_bounds__(ATT_SPLIT_WARPS * 32) attn_split_kernel(
    const float* P, int ldp, const uint16_t* kc, const uint16_t* vc, int max_ctx, int nq,
    int nkv, int pos0, int nsplit, float* part) {
  constexpr int EPL = HD / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sidx = blockIdx.x * ATT_SPLIT_WARPS + warp;
  const int h = blockIdx.y, t = blockIdx.z;
  if (sidx >= nsplit) return;
  const int g = h / (nq / nkv);
  const int nkeys = pos0 + t + 1;
  const int k0 = sidx * ATT_SPLIT_LEN, k1 = min(k0 + ATT_SPLIT_LEN, nkeys);
  float* out = part + ((size_t(t) * nq + h) * nsplit + sidx) * (HD + 2);
  float q[EPL];
  const float* qrow = P + size_t(t) * ldp + h * HD;
#pragma unroll
  for (int e = 0; e < EPL; ++e) q[e] = qrow[lane * EPL + e];
  const float scale = 1.0f / sqrtf(float(HD));
  const uint16_t* K = kc + size_t(g) * max_ctx * HD;
  const uint16_t* V = vc + size_t(g) * max_ctx * HD;
  float m = -INFINITY, l = 0.f, acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  constexpr int KB = 4;
  for (int j0 = k0; j0 < k1; j0 += KB) {
    float kf[KB][EPL], vf[KB][EPL], sc[KB];
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      const int j = min(j0 + u, k1 - 1);
      load_bf16_row<EPL>(K + size_t(j) * HD + lane * EPL, kf[u]);
      load_bf16_row<EPL>(V + size_t(j) * HD + lane * EPL, vf[u]);
    }
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      sc[u] = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) sc[u] = fmaf(q[e], kf[u][e], sc[u]);
    }
#pragma unroll
    for (int u = 0; u < KB; ++u) sc[u] = warp_sum(sc[u]) * scale;
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      if (j0 + u < k1) {
        const float mn = fmaxf(m, sc[u]);
        const float corr = expf(m - mn), p = expf(sc[u] - mn);
        l = l * corr + p;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = fmaf(p, vf[u][e], acc[e] * corr);
        m = mn;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) out[lane * EPL + e] = acc[e];
  if (lane == 0) {
    out[HD] = m;  // -inf when the range holds no key of this query
    out[HD + 1] = l;
  }
}

// o[t][h] = sum_s e^(m_s - M) acc_s / sum_s e^(m_s - M) l_s, written as split
// bf16 operands for the output-projection GEMM.  grid (nq, T), HD threads.
template <int HD>
__global__ void attn_merge_kernel(const float* part, int nq, int nsplit, uint16_t* Ob, int ldob,
                                  size_t lo, float* Of) {
  griddep_launch_dependents();
  const int h = blockIdx.x, t = blockIdx.y, i = threadIdx.x;
  const float* base = part + (size_t(t) * nq + h) * nsplit * (HD + 2);
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, base[size_t(s) * (HD + 2) + HD]);
  float den = 0.f, num = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float* ps = base + size_t(s) * (HD + 2);
    const float ls = ps[HD + 1];
    if (ls > 0.f) {
      const float wgt = expf(ps[HD] - M);
      den = fmaf(wgt, ls, den);
      num = fmaf(wgt, ps[i], num);
    }
  }
  if (Of)
    Of[size_t(t) * ldob + h * HD + i] = num / den;  // fp32 rows of the same width
  else
    store_split(Ob + size_t(t) * ldob + h * HD + i, lo, num / den);
}

}  // namespace pf
}  // namespace mk
