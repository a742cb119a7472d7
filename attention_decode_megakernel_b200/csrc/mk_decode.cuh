// mk_decode.cuh -- the single-launch decode kernel.
//
// One token's whole forward pass (embedding, every DeltaNet and attention
// layer with its MLP, final norm, tied LM head and greedy argmax) runs in ONE
// cooperative launch of a persistent grid with one CTA per SM, as in the
// launch post "OS Megakernel that match M5 Max Tok/w at 2x the Throughput on
// RTX 3090" (kernel bullet list: whole forward pass in one dispatch,
// cooperative grid sync instead of per-operation launches, bf16 weights with
// fp32 accumulation, fused QKV + RoPE + causal softmax + output projection).
//
// B200 structure (differs from the post's 3090 design):
//  * Each CTA owns a balanced slice of every phase (rows of each matrix,
//    rows of the recurrent state, a split of the KV cache).  The slices are
//    known at launch, so one producer warp walks the CTA's whole per-token
//    byte stream and keeps a 12 x 16 KB shared-memory ring full with bulk
//    TMA copies (cp.async.bulk + mbarrier complete_tx).  It never waits on a
//    grid barrier: weights, the previous token's state rows and the cached
//    KV positions of the next phases keep streaming from HBM while the
//    consumer warps wait for the rest of the grid.
//  * Eight consumer warps turn each chunk into results: warp-per-row bf16
//    GEMV against an fp32 activation vector held in registers, the gated
//    delta-rule row update, split-K flash-decode attention with an
//    online softmax and a last-CTA merge.  Phases that need the whole of the
//    previous phase's output are separated by a grid barrier on a gpu-scope
//    counter (release add / acquire poll), five per layer.
//  * Every wait is bounded by %globaltimer; on expiry the kernel records
//    MK_ERR_TIMEOUT, runs the rest of its schedule without work, lets its
//    in-flight copies land and returns.
#pragma once
#include "mk_model.cuh"
#include "mk_ptx.cuh"

namespace mk {

constexpr int NCW = 8;                  // consumer warps
constexpr int NCT = NCW * 32;           // consumer threads
constexpr int NTHR = NCT + 32;          // + producer warp
constexpr int SLOT = 16384;             // ring slot bytes
constexpr int NSLOT = 12;               // ring slots
constexpr int ATT_MIN_POS = 64;         // fewest positions per attention split
constexpr int XREG_VEC = 8;             // activation vectors (8 floats) per lane held in registers

enum PhaseKind { PH_DN_IN, PH_DN_ST, PH_OUT, PH_Q, PH_K, PH_V, PH_ATT, PH_GU, PH_DOWN, PH_LM };

struct StepArgs {
  const DevModel* m;
  int pos;            // position of this token
  int token;          // input token when tok_src == 0
  int tok_src;        // 1: take the token from amax[amax_in]
  int amax_in, amax_out;
  int st_buf;         // state buffer index
  float* logits;      // [V] (never NULL: scratch when the caller wants none)
  int32_t* tok_out;   // receives the argmax token (may be NULL)
  float* hidden;      // [n_layers][H] per-layer residual dump (may be NULL)
  unsigned bar_base;  // grid-barrier counter value at launch
  int fail_barrier;   // debug: barrier index that can never complete (-1 = none)
  long long wait_ns;  // bound of every device-side wait
};

// Shared memory carve-up (dynamic).
struct __align__(16) SmemTail {
  uint64_t full[NSLOT];
  uint64_t empty[NSLOT];
  float red[32];
  float rope_cos[128], rope_sin[128];
  int abort_flag;
  int flag;
  int token;
  unsigned long long best;
};

template <int DK, int HD, int GQ>
struct Cfg {
  static constexpr int EPL_S = DK / 32;  // state elements per lane
  static constexpr int EPL_A = HD / 32;  // head elements per lane
  static constexpr int GMAX = GQ;        // query heads per KV head
  // union region (bytes): activation vector | DeltaNet head cache | attention scratch
  static constexpr int XIN_FLOATS = 4096;
  static constexpr int DNC_HEADS = 8;
  static constexpr int ATT_FLOATS = GMAX * HD * 2 + 2 * HD + NCW * GMAX * 2;
  static constexpr int UNION_FLOATS =
      XIN_FLOATS > ATT_FLOATS ? XIN_FLOATS : ATT_FLOATS;
  static constexpr size_t SMEM = size_t(NSLOT) * SLOT + sizeof(SmemTail) + UNION_FLOATS * 4 + 128;
};

struct PD {                 // one CTA's share of one phase
  const char* p0;           // plane 0 base (row 0 of the phase's row space)
  const char* p1;           // plane 1 base or nullptr
  uint32_t row_bytes;       // bytes of one row of one plane
  int r0, n;                // first row and number of rows of this CTA
  int rpc;                  // rows per chunk
  uint64_t pol;             // L2 policy of the copies
  int unit_g, unit_s, S;    // attention split of this CTA (unit_g < 0: none)
};

__device__ __forceinline__ void balanced(int n, int idx, int parts, int& a, int& b) {
  a = int((long long)n * idx / parts);
  b = int((long long)n * (idx + 1) / parts);
}

__device__ __forceinline__ int att_splits(const DevModel& M, int pos) {
  int ctx = pos + 1;
  int s = (ctx + ATT_MIN_POS - 1) / ATT_MIN_POS;
  int smax = M.ncta / M.nkv;
  return s < smax ? s : smax;
}

__device__ __forceinline__ PD describe(const DevModel& M, const StepArgs& a, int kind, int l,
                                       int gp, int cta, uint64_t pol_w, uint64_t pol_s) {
  PD d;
  d.p0 = d.p1 = nullptr;
  d.row_bytes = 16;
  d.pol = pol_w;
  d.unit_g = -1;
  d.unit_s = 0;
  d.S = 0;
  const DevLayer& L = M.layers[l];
  int idx = (cta + gp) % M.ncta;
  int r0 = 0, r1 = 0;
  switch (kind) {
    case PH_DN_IN:
      balanced(M.rin, idx, M.ncta, r0, r1);
      d.p0 = (const char*)L.in_proj;
      d.row_bytes = M.H * 2;
      break;
    case PH_DN_ST:
      balanced(M.nh * M.dv, idx, M.ncta, r0, r1);
      d.p0 = (const char*)(M.dn_state[a.st_buf] + size_t(L.sub) * M.nh * M.dv * M.dk);
      d.row_bytes = M.dk * 4;
      d.pol = pol_s;
      break;
    case PH_OUT:
      balanced(M.H, idx, M.ncta, r0, r1);
      d.p0 = (const char*)(L.is_attn ? L.w_o : L.out_proj);
      d.row_bytes = (L.is_attn ? M.nq * M.hd : M.nh * M.dv) * 2;
      break;
    case PH_Q:
      balanced(M.nq * M.hd, idx, M.ncta, r0, r1);
      d.p0 = (const char*)L.w_q;
      d.row_bytes = M.H * 2;
      break;
    case PH_K:
      balanced(M.nkv * M.hd, idx, M.ncta, r0, r1);
      d.p0 = (const char*)L.w_k;
      d.row_bytes = M.H * 2;
      break;
    case PH_V:
      balanced(M.nkv * M.hd, idx, M.ncta, r0, r1);
      d.p0 = (const char*)L.w_v;
      d.row_bytes = M.H * 2;
      break;
    case PH_GU:
      balanced(M.I, idx, M.ncta, r0, r1);
      d.p0 = (const char*)L.w_gate;
      d.p1 = (const char*)L.w_up;
      d.row_bytes = M.H * 2;
      break;
    case PH_DOWN:
      balanced(M.H, idx, M.ncta, r0, r1);
      d.p0 = (const char*)L.w_down;
      d.row_bytes = M.I * 2;
      break;
    case PH_LM:
      balanced(M.V, idx, M.ncta, r0, r1);
      d.p0 = (const char*)M.embed;
      d.row_bytes = M.H * 2;
      break;
    case PH_ATT: {
      int S = att_splits(M, a.pos);
      d.S = S;
      d.row_bytes = M.hd * 2;
      d.pol = pol_s;
      if (cta < M.nkv * S) {
        int g = cta / S, s = cta % S;
        d.unit_g = g;
        d.unit_s = s;
        balanced(a.pos + 1, s, S, r0, r1);
        if (r1 > a.pos) r1 = a.pos;  // the new position is not in the cache yet
        size_t base = (size_t(L.sub) * M.nkv + g) * M.max_ctx * M.hd;
        d.p0 = (const char*)(M.kc + base);
        d.p1 = (const char*)(M.vc + base);
      }
      break;
    }
  }
  d.r0 = r0;
  d.n = r1 > r0 ? r1 - r0 : 0;
  d.rpc = SLOT / ((d.p1 ? 2 : 1) * int(d.row_bytes));
  return d;
}

// Phase sequence of one layer.
__device__ __forceinline__ int layer_phases(const DevLayer& L, int* kinds) {
  if (L.is_attn) {
    kinds[0] = PH_Q; kinds[1] = PH_K; kinds[2] = PH_V; kinds[3] = PH_ATT;
    kinds[4] = PH_OUT; kinds[5] = PH_GU; kinds[6] = PH_DOWN;
    return 7;
  }
  kinds[0] = PH_DN_IN; kinds[1] = PH_DN_ST; kinds[2] = PH_OUT; kinds[3] = PH_GU; kinds[4] = PH_DOWN;
  return 5;
}
__device__ __forceinline__ bool has_grid_barrier(int kind) {
  return !(kind == PH_Q || kind == PH_K || kind == PH_LM);
}

// ----------------------------------------------------------------------------
// bounded waits
// ----------------------------------------------------------------------------
__device__ __forceinline__ void record_error(const DevModel& M, int code) {
  atomicCAS(M.err, 0, code);
}

__device__ __forceinline__ bool aborted(SmemTail* t) { return *(volatile int*)&t->abort_flag != 0; }

// Returns false (and leaves the CTA in abort mode) when the wait gave up.
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, SmemTail* t,
                                             const DevModel& M, long long wait_ns) {
  if (aborted(t)) return false;
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t start = global_ns();
  for (int it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31) == 0) {
      if (*(volatile int*)&t->abort_flag) return false;
      if (global_ns() - start > uint64_t(wait_ns)) {
        record_error(M, MK_ERR_TIMEOUT);
        *(volatile int*)&t->abort_flag = 1;
        return false;
      }
    }
  }
}

// Grid barrier number `k` of this launch (one thread per CTA).
__device__ __forceinline__ bool grid_barrier(const DevModel& M, const StepArgs& a, int k,
                                             SmemTail* t) {
  if (aborted(t)) return false;
  __threadfence();
  red_add_release_gpu(M.bar, 1u);
  unsigned target = a.bar_base + unsigned(k + 1) * unsigned(M.ncta);
  if (k == a.fail_barrier) target += 1u;  // debug: one arrival more than exists
  uint64_t start = global_ns();
  for (int it = 0;; ++it) {
    unsigned v = ld_acquire_gpu(M.bar);
    if (int(v - target) >= 0) return true;
    if ((it & 15) == 15) {
      if (ld_relaxed_gpu(M.err) != 0) {
        *(volatile int*)&t->abort_flag = 1;
        return false;
      }
      if (global_ns() - start > uint64_t(a.wait_ns)) {
        record_error(M, MK_ERR_TIMEOUT);
        *(volatile int*)&t->abort_flag = 1;
        return false;
      }
    }
  }
}

// ----------------------------------------------------------------------------
// GEMV helpers (warp per row)
// ----------------------------------------------------------------------------
__device__ __forceinline__ void load_xregs(float (&xr)[XREG_VEC][8], const float* xin, int nvec,
                                           int lane) {
#pragma unroll
  for (int v = 0; v < XREG_VEC; ++v) {
    int idx = v * 32 + lane;
    if (idx < nvec) {
      float4 p = reinterpret_cast<const float4*>(xin)[idx * 2];
      float4 q = reinterpret_cast<const float4*>(xin)[idx * 2 + 1];
      xr[v][0] = p.x; xr[v][1] = p.y; xr[v][2] = p.z; xr[v][3] = p.w;
      xr[v][4] = q.x; xr[v][5] = q.y; xr[v][6] = q.z; xr[v][7] = q.w;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) xr[v][e] = 0.f;
    }
  }
}

__device__ __forceinline__ void fma8(const uint4 w, const float* x, float& a0, float& a1,
                                     float& a2, float& a3) {
  a0 = fmaf(bf_lo(w.x), x[0], a0);
  a1 = fmaf(bf_hi(w.x), x[1], a1);
  a2 = fmaf(bf_lo(w.y), x[2], a2);
  a3 = fmaf(bf_hi(w.y), x[3], a3);
  a0 = fmaf(bf_lo(w.z), x[4], a0);
  a1 = fmaf(bf_hi(w.z), x[5], a1);
  a2 = fmaf(bf_lo(w.w), x[6], a2);
  a3 = fmaf(bf_hi(w.w), x[7], a3);
}

// Partial dot of one bf16 row (nvec 16-byte vectors in shared memory) with
// the register-resident activation; the caller reduces over the warp.
__device__ __forceinline__ float row_dot_regs(const uint4* w, const float (&xr)[XREG_VEC][8],
                                              int nvec, int lane) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int v = 0; v < XREG_VEC; ++v) {
    int idx = v * 32 + lane;
    if (idx < nvec) fma8(w[idx], xr[v], a0, a1, a2, a3);
  }
  return (a0 + a1) + (a2 + a3);
}

// Same with the activation read from shared memory (long rows).
__device__ __forceinline__ float row_dot_smem(const uint4* w, const float* xin, int nvec,
                                              int lane) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  for (int idx = lane; idx < nvec; idx += 32) {
    float x[8];
    float4 p = reinterpret_cast<const float4*>(xin)[idx * 2];
    float4 q = reinterpret_cast<const float4*>(xin)[idx * 2 + 1];
    x[0] = p.x; x[1] = p.y; x[2] = p.z; x[3] = p.w;
    x[4] = q.x; x[5] = q.y; x[6] = q.z; x[7] = q.w;
    fma8(w[idx], x, a0, a1, a2, a3);
  }
  return (a0 + a1) + (a2 + a3);
}

// ----------------------------------------------------------------------------
// consumer pre-phase builders (all NCT consumer threads)
// ----------------------------------------------------------------------------
// xin = RMSNorm(src) * gain; src is the fp32 residual (gpu-coherent loads) or,
// for the first layer, the bf16 embedding row of the token.
__device__ void build_rmsnorm(float* xin, const float* src, const uint16_t* emb_row,
                              const uint16_t* gain, int H, float eps, SmemTail* t, int tid) {
  float ss = 0.f;
  for (int i = tid; i < H; i += NCT) {
    float v = emb_row ? bf2f(emb_row[i]) : __ldcg(src + i);
    xin[i] = v;
    ss = fmaf(v, v, ss);
  }
  ss = warp_sum(ss);
  if ((tid & 31) == 0) t->red[tid >> 5] = ss;
  named_sync(1, NCT);
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < NCW; ++w) tot += t->red[w];
  float inv = 1.0f / sqrtf(tot / float(H) + eps);
  for (int i = tid; i < H; i += NCT) xin[i] = xin[i] * inv * bf2f(gain[i]);
  named_sync(1, NCT);
}

__device__ void build_copy(float* xin, const float* src, int n, int tid) {
  for (int i = tid; i < n; i += NCT) xin[i] = __ldcg(src + i);
  named_sync(1, NCT);
}

// xin[h*dv+i] = RMSNorm_dv(o_h)_i * out_norm_i * SiLU(z_h,i): the gated
// output norm of the DeltaNet layer (warp per head).
template <int DK>
__device__ void build_gated_norm(float* xin, const DevModel& M, const DevLayer& L, int tid) {
  constexpr int EPL = DK / 32;  // dv == dk
  int warp = tid >> 5, lane = tid & 31;
  const float* z = M.inp + M.ch;
  for (int h = warp; h < M.nh; h += NCW) {
    float o[EPL];
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      o[e] = __ldcg(M.dno + h * M.dv + lane * EPL + e);
      ss = fmaf(o[e], o[e], ss);
    }
    ss = warp_sum(ss);
    float inv = 1.0f / sqrtf(ss / float(M.dv) + M.eps);
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      int i = lane * EPL + e;
      float zz = __ldcg(z + h * M.dv + i);
      xin[h * M.dv + i] = o[e] * inv * bf2f(L.out_norm[i]) * siluf_(zz);
    }
  }
  named_sync(1, NCT);
}

// ----------------------------------------------------------------------------
// consumer chunk loop: wait for each chunk of the CTA's share of a phase,
// hand this warp's rows to `fn(row, plane0_row, plane1_row)`, release the slot
// ----------------------------------------------------------------------------
// (A macro rather than a function taking a lambda: the body must be inlined
// so that register-resident activations and accumulators stay in registers.)
// Uses the enclosing scope's M, a, t, ring, g, warp, lane; the body sees
// `row`, `p0` (plane-0 row in shared memory) and `p1` (plane-1 row).
#define MK_CHUNK_LOOP(d, ...)                                                          \
  do {                                                                                 \
    int local_ = 0;                                                                    \
    for (int r_ = (d).r0; r_ < (d).r0 + (d).n; r_ += (d).rpc, ++g, local_ += (d).rpc) { \
      const int slot_ = int(g % NSLOT);                                                \
      const bool ok_ = bounded_wait(&t->full[slot_], (g / NSLOT) & 1, t, M, a.wait_ns); \
      if (ok_) {                                                                       \
        const int nr_ = min((d).rpc, (d).r0 + (d).n - r_);                             \
        const unsigned char* base_ = ring + size_t(slot_) * SLOT;                      \
        for (int i_ = (warp - (local_ % NCW) + NCW) % NCW; i_ < nr_; i_ += NCW) {      \
          const int row = r_ + i_;                                                     \
          const unsigned char* p0 = base_ + size_t(i_) * (d).row_bytes;                \
          const unsigned char* p1 = base_ + size_t((d).rpc + i_) * (d).row_bytes;      \
          (void)row; (void)p0; (void)p1;                                               \
          __VA_ARGS__                                                                  \
        }                                                                              \
      }                                                                                \
      __syncwarp();                                                                    \
      if (lane == 0) mbar_arrive(&t->empty[slot_]);                                    \
    }                                                                                  \
  } while (0)

// ----------------------------------------------------------------------------
// gated delta rule on this CTA's rows of the state (one layer, one token)
// ----------------------------------------------------------------------------
template <int DK>
__device__ __forceinline__ void dn_state_phase(const DevModel& M, const StepArgs& a,
                                               const DevLayer& L, const PD& d, uint32_t& g,
                                               unsigned char* ring, SmemTail* t, float* uni,
                                               bool dry, int tid, int warp, int lane) {
  constexpr int EPL = DK / 32;
  constexpr int stride = 2 * DK + 4;  // head cache: [q(dk) | k(dk) | beta, alpha, k.q, -]
  int h_first = 0;
  if (!dry && d.n > 0) {
    h_first = d.r0 / M.dv;
    const int h_last = (d.r0 + d.n - 1) / M.dv;
    for (int hh = warp; hh <= h_last - h_first; hh += NCW) {
      const int h = h_first + hh;
      float qv[EPL], kv[EPL];
      float sq = 0.f, sk = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        qv[e] = __ldcg(M.inp + h * DK + lane * EPL + e);
        kv[e] = __ldcg(M.inp + M.nh * DK + h * DK + lane * EPL + e);
        sq = fmaf(qv[e], qv[e], sq);
        sk = fmaf(kv[e], kv[e], sk);
      }
      sq = warp_sum(sq);
      sk = warp_sum(sk);
      // q, k L2-normalised (eps 1e-6 inside the root); q also scaled by dk^-1/2
      const float iq = 1.0f / sqrtf(sq + 1e-6f) / sqrtf(float(DK));
      const float ik = 1.0f / sqrtf(sk + 1e-6f);
      float kq = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        qv[e] *= iq;
        kv[e] *= ik;
        kq = fmaf(kv[e], qv[e], kq);
        uni[hh * stride + lane * EPL + e] = qv[e];
        uni[hh * stride + DK + lane * EPL + e] = kv[e];
      }
      kq = warp_sum(kq);
      if (lane == 0) {
        const float b = __ldcg(M.inp + M.ch + M.nh * M.dv + h);
        const float aa = __ldcg(M.inp + M.ch + M.nh * M.dv + M.nh + h);
        uni[hh * stride + 2 * DK + 0] = sigmoidf_(b);                                   // beta
        uni[hh * stride + 2 * DK + 1] = expf(-expf(L.A_log[h]) * softplusf_(aa + L.dt_bias[h]));  // alpha
        uni[hh * stride + 2 * DK + 2] = kq;
      }
    }
  }
  named_sync(1, NCT);
  float* st = M.dn_state[a.st_buf] + size_t(L.sub) * M.nh * M.dv * DK;
  MK_CHUNK_LOOP(d, 
    const int h = row / M.dv, iv = row % M.dv;
    const float* hc = uni + (h - h_first) * stride;
    const float* sr = reinterpret_cast<const float*>(p0) + lane * EPL;
    float sv[EPL], kv[EPL];
    float s_k = 0.f, s_q = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      sv[e] = sr[e];
      kv[e] = hc[DK + lane * EPL + e];
      s_k = fmaf(sv[e], kv[e], s_k);
      s_q = fmaf(sv[e], hc[lane * EPL + e], s_q);
    }
    s_k = warp_sum(s_k);
    s_q = warp_sum(s_q);
    const float beta = hc[2 * DK], alpha = hc[2 * DK + 1], kq = hc[2 * DK + 2];
    const float vi = __ldcg(M.inp + 2 * M.nh * DK + h * M.dv + iv);
    const float u = beta * (vi - alpha * s_k);  // S' = alpha S + u k^T
    float* dst = st + size_t(row) * DK + lane * EPL;
    if constexpr (EPL == 4) {
      *reinterpret_cast<float4*>(dst) =
          make_float4(fmaf(alpha, sv[0], u * kv[0]), fmaf(alpha, sv[1], u * kv[1]),
                      fmaf(alpha, sv[2], u * kv[2]), fmaf(alpha, sv[3], u * kv[3]));
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) dst[e] = fmaf(alpha, sv[e], u * kv[e]);
    }
    if (lane == 0) M.dno[row] = fmaf(alpha, s_q, u * kq);  // o_i = S'_i . q
  );
}

// One key/value row into a warp's online-softmax state for G query heads
// (this lane's EPL elements of the row).
template <int G, int EPL>
__device__ __forceinline__ void att_consume(float (&am)[G], float (&al)[G], float (&acc)[G][EPL],
                                            const float (&qr)[G][EPL], const float* kf,
                                            const float* vf, float scale) {
#pragma unroll
  for (int j = 0; j < G; ++j) {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) s = fmaf(qr[j][e], kf[e], s);
    s = warp_sum(s) * scale;
    const float mn = fmaxf(am[j], s);
    const float corr = expf(am[j] - mn);
    const float pr = expf(s - mn);
    al[j] = al[j] * corr + pr;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[j][e] = fmaf(pr, vf[e], acc[j][e] * corr);
    am[j] = mn;
  }
}

// ----------------------------------------------------------------------------
// split-K flash-decode attention for one KV group and position range
// ----------------------------------------------------------------------------
template <int HD, int GQ>
__device__ __forceinline__ void attention_phase(const DevModel& M, const StepArgs& a,
                                                const DevLayer& L, const PD& d, uint32_t& g,
                                                unsigned char* ring, SmemTail* t, float* uni,
                                                bool dry, int tid, int warp, int lane) {
  constexpr int EPL = HD / 32;
  constexpr int G = GQ;
  float* att_q = uni;                   // [G][HD] rotated queries
  float* att_acc = uni + G * HD;        // [G][HD] CTA accumulator
  float* att_kn = uni + 2 * G * HD;     // [HD] new key (bf16-rounded)
  float* att_vn = att_kn + HD;          // [HD] new value
  float* att_ml = att_vn + HD;          // [NCW][G][2] warp (m, l)
  const bool unit = d.unit_g >= 0;
  const bool last = unit && d.unit_s == d.S - 1;
  const int gidx = d.unit_g;
  if (unit && !dry) {
    const int half = HD / 2;
    for (int i = tid; i < G * half; i += NCT) {
      const int j = i / half, c = i % half;
      const float* qh = M.qkv + (gidx * G + j) * HD;
      const float x0 = __ldcg(qh + c), x1 = __ldcg(qh + c + half);
      const float cs = t->rope_cos[c], sn = t->rope_sin[c];
      att_q[j * HD + c] = x0 * cs - x1 * sn;
      att_q[j * HD + c + half] = x1 * cs + x0 * sn;
    }
    for (int i = tid; i < G * HD; i += NCT) att_acc[i] = 0.f;
    if (last) {
      // RoPE the new key, store K/V at `pos` in bf16, keep the rounded values
      const float* kr = M.qkv + M.nq * HD + gidx * HD;
      const float* vr = M.qkv + (M.nq + M.nkv) * HD + gidx * HD;
      const size_t cofs = ((size_t(L.sub) * M.nkv + gidx) * M.max_ctx + a.pos) * HD;
      for (int c = tid; c < half; c += NCT) {
        const float x0 = __ldcg(kr + c), x1 = __ldcg(kr + c + half);
        const float cs = t->rope_cos[c], sn = t->rope_sin[c];
        const uint16_t b0 = f2bf(x0 * cs - x1 * sn), b1 = f2bf(x1 * cs + x0 * sn);
        M.kc[cofs + c] = b0;
        M.kc[cofs + c + half] = b1;
        att_kn[c] = bf2f(b0);
        att_kn[c + half] = bf2f(b1);
      }
      for (int c = tid; c < HD; c += NCT) {
        const uint16_t b = f2bf(__ldcg(vr + c));
        M.vc[cofs + c] = b;
        att_vn[c] = bf2f(b);
      }
    }
  }
  named_sync(1, NCT);
  // per-warp online-softmax state over this warp's positions
  float am[G], al[G], acc[G][EPL], qr[G][EPL];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    am[j] = -INFINITY;
    al[j] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      acc[j][e] = 0.f;
      qr[j][e] = (unit && !dry) ? att_q[j * HD + lane * EPL + e] : 0.f;
    }
  }
  const float scale = 1.0f / sqrtf(float(HD));
  MK_CHUNK_LOOP(d, 
    const uint16_t* k16 = reinterpret_cast<const uint16_t*>(p0) + lane * EPL;
    const uint16_t* v16 = reinterpret_cast<const uint16_t*>(p1) + lane * EPL;
    float kf[EPL], vf[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      kf[e] = bf2f(k16[e]);
      vf[e] = bf2f(v16[e]);
    }
    att_consume<G, EPL>(am, al, acc, qr, kf, vf, scale);
  );
  const bool dry_post = named_sync_or(1, NCT, aborted(t));
  if (!unit || dry_post) return;
  // the new position (not in the cache at launch) goes to the next warp in turn
  if (last && warp == (d.n % NCW)) {
    float kf[EPL], vf[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      kf[e] = att_kn[lane * EPL + e];
      vf[e] = att_vn[lane * EPL + e];
    }
    att_consume<G, EPL>(am, al, acc, qr, kf, vf, scale);
  }
  // combine the warps' (m, l, acc) into one partial for this split
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < G; ++j) {
      att_ml[(warp * G + j) * 2 + 0] = am[j];
      att_ml[(warp * G + j) * 2 + 1] = al[j];
    }
  }
  named_sync(1, NCT);
  // fixed warp order (deterministic): warp w adds its rescaled accumulator
  float fw[G];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    float mx = -INFINITY;
    for (int w = 0; w < NCW; ++w) mx = fmaxf(mx, att_ml[(w * G + j) * 2]);
    fw[j] = al[j] > 0.f ? expf(am[j] - mx) : 0.f;
  }
  for (int w = 0; w < NCW; ++w) {
    if (warp == w) {
#pragma unroll
      for (int j = 0; j < G; ++j)
#pragma unroll
        for (int e = 0; e < EPL; ++e) att_acc[j * HD + lane * EPL + e] += fw[j] * acc[j][e];
    }
    named_sync(1, NCT);
  }
  float* pbase = M.part + (size_t(gidx) * kMaxCtas + d.unit_s) * G * (HD + 2);
  for (int i = tid; i < G * HD; i += NCT) pbase[(i / HD) * (HD + 2) + (i % HD)] = att_acc[i];
  if (tid < G) {
    float mx = -INFINITY, ls = 0.f;
    for (int w = 0; w < NCW; ++w) mx = fmaxf(mx, att_ml[(w * G + tid) * 2]);
    for (int w = 0; w < NCW; ++w) {
      const float lw = att_ml[(w * G + tid) * 2 + 1];
      if (lw > 0.f) ls += lw * expf(att_ml[(w * G + tid) * 2] - mx);
    }
    pbase[tid * (HD + 2) + HD] = mx;
    pbase[tid * (HD + 2) + HD + 1] = ls;
  }
  __threadfence();
  named_sync(1, NCT);
  if (tid == 0) {
    unsigned* tk = M.tickets + L.sub * M.nkv + gidx;
    const unsigned prev = atomicAdd(tk, 1u);
    t->flag = (prev == unsigned(d.S - 1)) ? 1 : 0;
    if (t->flag) atomicExch(tk, 0u);
  }
  named_sync(1, NCT);
  if (t->flag) {
    // last split of this KV group: merge the S partials into atto
    __threadfence();
    for (int i = tid; i < G * HD; i += NCT) {
      const int j = i / HD, e = i % HD;
      float mx = -INFINITY;
      for (int s = 0; s < d.S; ++s)
        mx = fmaxf(mx, __ldcg(M.part + (size_t(gidx) * kMaxCtas + s) * G * (HD + 2) +
                              j * (HD + 2) + HD));
      float num = 0.f, den = 0.f;
      for (int s = 0; s < d.S; ++s) {
        const float* pb = M.part + (size_t(gidx) * kMaxCtas + s) * G * (HD + 2) + j * (HD + 2);
        const float f = expf(__ldcg(pb + HD) - mx);
        num = fmaf(f, __ldcg(pb + e), num);
        den = fmaf(f, __ldcg(pb + HD + 1), den);
      }
      M.atto[(gidx * G + j) * HD + e] = num / den;
    }
  }
}

// ----------------------------------------------------------------------------
// the kernel
// ----------------------------------------------------------------------------
template <int DK, int HD, int GQ>
__global__ void __launch_bounds__(NTHR, 1) decode_kernel(const StepArgs a) {
  using C = Cfg<DK, HD, GQ>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* ring = smem_raw;
  SmemTail* t = reinterpret_cast<SmemTail*>(smem_raw + size_t(NSLOT) * SLOT);
  float* uni = reinterpret_cast<float*>(smem_raw + size_t(NSLOT) * SLOT + sizeof(SmemTail));

  const DevModel& M = *a.m;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;

  if (tid == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&t->full[s], 1);
      mbar_init(&t->empty[s], NCW);
    }
    t->abort_flag = 0;
    t->best = 0ull;
    int tok = a.token;
    if (a.tok_src) tok = int(0xFFFFFFFFu - uint32_t(__ldcg(&M.amax[a.amax_in]) & 0xFFFFFFFFull));
    if (tok < 0 || tok >= M.V) tok = 0;
    t->token = tok;
    if (cta == 0) M.amax[a.amax_out] = 0ull;  // reset before any CTA's atomicMax
    fence_barrier_init();
  }
  // RoPE table for this position (angles in double: pos * theta^(-2i/hd)).
  for (int i = tid; i < HD / 2; i += NTHR) {
    double inv_freq = pow(double(M.theta), -2.0 * double(i) / double(HD));
    double s, c;
    sincos(double(a.pos) * inv_freq, &s, &c);
    t->rope_cos[i] = float(c);
    t->rope_sin[i] = float(s);
  }
  __syncthreads();

  const uint64_t pol_w = policy_evict_first();
  const uint64_t pol_s = policy_evict_last();

  // ======================= producer warp ====================================
  if (warp == NCW) {
    if (lane != 0) return;
    uint32_t g = 0;
    int gp = 0;
    int kinds[8];
    for (int l = 0; l <= M.n_layers && !aborted(t); ++l) {
      int np;
      if (l < M.n_layers) np = layer_phases(M.layers[l], kinds);
      else { kinds[0] = PH_LM; np = 1; }
      for (int p = 0; p < np && !aborted(t); ++p, ++gp) {
        PD d = describe(M, a, kinds[p], l < M.n_layers ? l : 0, gp, cta, pol_w, pol_s);
        for (int r = d.r0; r < d.r0 + d.n; r += d.rpc, ++g) {
          int slot = int(g % NSLOT);
          if (g >= NSLOT && !bounded_wait(&t->empty[slot], ((g / NSLOT) - 1) & 1, t, M, a.wait_ns))
            break;
          int nr = min(d.rpc, d.r0 + d.n - r);
          uint32_t bytes = uint32_t(nr) * d.row_bytes;
          unsigned char* dst = ring + size_t(slot) * SLOT;
          mbar_arrive_expect_tx(&t->full[slot], bytes * (d.p1 ? 2u : 1u));
          bulk_g2s(dst, d.p0 + size_t(r) * d.row_bytes, bytes, &t->full[slot], d.pol);
          if (d.p1)
            bulk_g2s(dst + size_t(d.rpc) * d.row_bytes, d.p1 + size_t(r) * d.row_bytes, bytes,
                     &t->full[slot], d.pol);
        }
      }
    }
    // Let every copy still in flight land before the CTA may exit.
    uint32_t first = g > uint32_t(NSLOT) ? g - NSLOT : 0u;
    for (uint32_t q = first; q < g; ++q) {
      uint64_t start = global_ns();
      while (!mbar_try_wait(&t->full[q % NSLOT], (q / NSLOT) & 1)) {
        if (global_ns() - start > uint64_t(a.wait_ns)) break;
      }
    }
    return;
  }

  // ======================= consumer warps ===================================
  const int tok = t->token;
  const uint16_t* emb_row = M.embed + size_t(tok) * M.H;
  uint32_t g = 0;  // chunk counter (same order as the producer)
  int gp = 0, nbar = 0;
  float best_v = -INFINITY;
  int best_i = 0x7FFFFFFF;
  int kinds[8];
  bool first_residual = true;

  for (int l = 0; l <= M.n_layers; ++l) {
    const bool lm = (l == M.n_layers);
    const DevLayer& L = M.layers[lm ? 0 : l];
    int np;
    if (!lm) np = layer_phases(L, kinds);
    else { kinds[0] = PH_LM; np = 1; }

    for (int p = 0; p < np; ++p, ++gp) {
      const int kind = kinds[p];
      const PD d = describe(M, a, kind, lm ? 0 : l, gp, cta, pol_w, pol_s);
      // uniform across the consumer warps (also orders the previous phase)
      const bool dry = named_sync_or(1, NCT, aborted(t));
      const int row_vecs = int(d.row_bytes / 16);
      switch (kind) {
        case PH_DN_IN: {
          if (!dry) build_rmsnorm(uni, M.x, l == 0 ? emb_row : nullptr, L.attn_norm, M.H, M.eps, t, tid);
          float xr[XREG_VEC][8];
          load_xregs(xr, uni, row_vecs, lane);
          const float4* conv_st = reinterpret_cast<const float4*>(M.conv_state[a.st_buf]);
          float4* conv_wr = reinterpret_cast<float4*>(M.conv_state[a.st_buf]);
          MK_CHUNK_LOOP(d, 
            float y = warp_sum(row_dot_regs(reinterpret_cast<const uint4*>(p0), xr, row_vecs, lane));
            if (lane == 0) {
              if (row < M.ch) {
                // causal conv (taps u_{t-3}, u_{t-2}, u_{t-1}, u_t) + SiLU, shift the history
                const size_t ci = size_t(L.sub) * M.ch + row;
                float4 s = conv_st[ci];
                uint2 wc = *reinterpret_cast<const uint2*>(L.conv_w + size_t(row) * 4);
                float c = bf_lo(wc.x) * s.x + bf_hi(wc.x) * s.y + bf_lo(wc.y) * s.z + bf_hi(wc.y) * y;
                conv_wr[ci] = make_float4(s.y, s.z, y, 0.f);
                M.inp[row] = siluf_(c);
              } else {
                M.inp[row] = y;
              }
            }
          );
          break;
        }
        case PH_Q:
        case PH_K:
        case PH_V: {
          if (kind == PH_Q && !dry)
            build_rmsnorm(uni, M.x, l == 0 ? emb_row : nullptr, L.attn_norm, M.H, M.eps, t, tid);
          float xr[XREG_VEC][8];
          load_xregs(xr, uni, row_vecs, lane);
          const int off = kind == PH_Q ? 0 : (kind == PH_K ? M.nq * HD : (M.nq + M.nkv) * HD);
          MK_CHUNK_LOOP(d, 
            float y = warp_sum(row_dot_regs(reinterpret_cast<const uint4*>(p0), xr, row_vecs, lane));
            if (lane == 0) M.qkv[off + row] = y;
          );
          break;
        }
        case PH_GU: {
          if (!dry) build_rmsnorm(uni, M.x, nullptr, L.mlp_norm, M.H, M.eps, t, tid);
          float xr[XREG_VEC][8];
          load_xregs(xr, uni, row_vecs, lane);
          MK_CHUNK_LOOP(d, 
            float yg = warp_sum(row_dot_regs(reinterpret_cast<const uint4*>(p0), xr, row_vecs, lane));
            float yu = warp_sum(row_dot_regs(reinterpret_cast<const uint4*>(p1), xr, row_vecs, lane));
            if (lane == 0) M.mlph[row] = siluf_(yg) * yu;
          );
          break;
        }
        case PH_OUT:
        case PH_DOWN: {
          if (!dry) {
            if (kind == PH_DOWN) build_copy(uni, M.mlph, M.I, tid);
            else if (L.is_attn) build_copy(uni, M.atto, M.nq * M.hd, tid);
            else build_gated_norm<DK>(uni, M, L, tid);
          }
          const bool first = kind == PH_OUT && first_residual;
          float* hid = kind == PH_DOWN ? a.hidden : nullptr;
          if (row_vecs <= XREG_VEC * 32) {
            float xr[XREG_VEC][8];
            load_xregs(xr, uni, row_vecs, lane);
            MK_CHUNK_LOOP(d, 
              float y = warp_sum(row_dot_regs(reinterpret_cast<const uint4*>(p0), xr, row_vecs, lane));
              if (lane == 0) {
                float xn = (first ? bf2f(emb_row[row]) : __ldcg(M.x + row)) + y;
                M.x[row] = xn;
                if (hid) hid[size_t(l) * M.H + row] = xn;
              }
            );
          } else {
            MK_CHUNK_LOOP(d, 
              float y = warp_sum(row_dot_smem(reinterpret_cast<const uint4*>(p0), uni, row_vecs, lane));
              if (lane == 0) {
                float xn = (first ? bf2f(emb_row[row]) : __ldcg(M.x + row)) + y;
                M.x[row] = xn;
                if (hid) hid[size_t(l) * M.H + row] = xn;
              }
            );
          }
          if (kind == PH_OUT) first_residual = false;
          break;
        }
        case PH_LM: {
          if (!dry) build_rmsnorm(uni, M.x, nullptr, M.final_norm, M.H, M.eps, t, tid);
          float xr[XREG_VEC][8];
          load_xregs(xr, uni, row_vecs, lane);
          float* logits = a.logits;
          MK_CHUNK_LOOP(d, 
            float y = warp_sum(row_dot_regs(reinterpret_cast<const uint4*>(p0), xr, row_vecs, lane));
            if (lane == 0) {
              logits[row] = y;
              if (y > best_v || (y == best_v && row < best_i)) { best_v = y; best_i = row; }
            }
          );
          break;
        }
        case PH_DN_ST:
          dn_state_phase<DK>(M, a, L, d, g, ring, t, uni, dry, tid, warp, lane);
          break;
        case PH_ATT:
          attention_phase<HD, GQ>(M, a, L, d, g, ring, t, uni, dry, tid, warp, lane);
          break;
        default:
          break;
      }

      if (has_grid_barrier(kind)) {
        named_sync(1, NCT);
        if (tid == 0) grid_barrier(M, a, nbar, t);
        ++nbar;
        named_sync(1, NCT);
      }
    }
  }

  // ---------------- argmax over the grid ----------------
  if (lane == 0 && best_i != 0x7FFFFFFF) atomicMax(&t->best, pack_argmax(best_v, best_i));
  named_sync(1, NCT);
  if (tid == 0 && !aborted(t)) {
    if (t->best) atomicMax(&M.amax[a.amax_out], t->best);
    __threadfence();
    unsigned* tk = M.tickets + M.n_attn * M.nkv;
    unsigned prev = atomicAdd(tk, 1u);
    if (prev == unsigned(M.ncta - 1)) {
      atomicExch(tk, 0u);
      __threadfence();
      unsigned long long v = atomicAdd(&M.amax[a.amax_out], 0ull);
      if (a.tok_out) *a.tok_out = int(0xFFFFFFFFu - uint32_t(v & 0xFFFFFFFFull));
    }
  }
}

}  // namespace mk
