// mk_decode.cuh -- the single-launch decode kernel.
//
// One token's whole forward pass (embedding, every DeltaNet and attention
// layer with its MLP, final norm, tied LM head and greedy argmax) runs in ONE
// cooperative launch of a persistent grid with one CTA per SM, as in the
// launch post "OS Megakernel that match M5 Max Tok/w at 2x the Throughput on
// RTX 3090" (kernel bullet list: whole forward pass in one dispatch, no
// per-operation launches, bf16 weights with fp32 accumulation, fused QKV +
// RoPE + causal softmax + output projection).
//
// B200 structure (differs from the post's 3090 design):
//  * Each CTA owns a balanced slice of every phase (rows of each matrix,
//    rows of the recurrent state, a split of the KV cache).  The slices are
//    known at launch, so one producer warp walks the CTA's whole per-token
//    byte stream and keeps a 3 x 64 KB shared-memory ring full with bulk TMA
//    copies (cp.async.bulk + mbarrier complete_tx).  It never waits for
//    other CTAs: weights, the previous token's state rows and cached KV
//    positions of later phases keep streaming while the consumers wait.
//  * Cross-CTA data travels as tagged words: every activation element another
//    CTA needs is stored as one 8-byte word {fp32 value, 32-bit tag}, the tag
//    naming the launch and the phase that produced it.  A consumer polls the
//    words it needs until all tags match, so one L2 round trip both
//    synchronises and delivers the vector; there is no grid barrier, no
//    fence and no counter on the data path.  (The post's cooperative grid
//    sync between layers is replaced by this data-driven wait.)
//  * Eleven consumer warps: bf16 GEMV rows (four per warp at a time) against
//    the fp32 activation vector in shared memory, the gated delta-rule row
//    update, split-K flash-decode attention with an online softmax and a
//    cooperative merge, SwiGLU, the tied LM head with a grid argmax.
//  * Every wait is bounded by %globaltimer; on expiry the kernel records
//    MK_ERR_TIMEOUT, runs the rest of its schedule without work, lets its
//    in-flight copies land and returns.
#pragma once
#include "mk_model.cuh"
#include "mk_ptx.cuh"

namespace mk {

constexpr int NCW = 11;                 // consumer warps (12 warps per CTA: 168 registers each)
constexpr int NCT = NCW * 32;           // consumer threads
constexpr int NTHR = NCT + 32;          // + producer warp
constexpr int SLOT = 65536;             // ring slot bytes (more rows per slot: more rows per warp)
constexpr int NSLOT = 3;                // ring slots
constexpr int ATT_MIN_POS = 32;         // fewest positions per attention split
constexpr int XRAW_MAX = 2048;          // largest hidden size (residual copy in shared memory)
constexpr int UNION_FLOATS = 4096;      // activation vector | head cache | attention scratch
constexpr int DN_HEADS_MAX = 4;         // heads one CTA's state rows may touch
constexpr int DN_ROWS_MAX = 256;        // state rows of one CTA
constexpr int CONV_ROWS_MAX = 256;      // in-projection rows of one CTA (conv staging)

// words per consumer thread when NCT threads gather n tagged values
constexpr int per_thread(int n) { return (n + NCT - 1) / NCT; }

enum PhaseKind { PH_DN_IN, PH_DN_ST, PH_OUT, PH_QKV, PH_ATT, PH_GU, PH_DOWN, PH_LM };

struct StepArgs {
  DevModel m;         // the engine (by value: read through the constant bank)
  int pos;            // position of this token
  int token;          // input token when tok_src == 0
  int tok_src;        // 1: take the token from amax[amax_in]
  int amax_in, amax_out;
  int st_buf;         // state buffer index
  float* logits;      // [V] (never NULL: scratch when the caller wants none)
  int32_t* tok_out;   // receives the argmax token (may be NULL)
  float* hidden;      // [n_layers][H] per-layer residual dump (may be NULL)
  uint32_t seq;       // launch sequence number, 1 .. 2^23-1 (tag = seq << 8 | phase)
  int fail_phase;     // debug: phase whose input tag can never match (-1 = none)
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
  static_assert(GQ * HD * 2 + 2 * HD + NCW * GQ * 2 <= UNION_FLOATS, "attention scratch");
  static_assert(DN_HEADS_MAX * (2 * DK + 4) + 2 * DN_HEADS_MAX * DK + DN_ROWS_MAX +
                    2 * DN_HEADS_MAX <= UNION_FLOATS,
                "state-phase scratch");
  static constexpr size_t SMEM =
      size_t(NSLOT) * SLOT + sizeof(SmemTail) + (UNION_FLOATS + XRAW_MAX) * 4 + 128;
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

// Not inlined: the producer's two cursors and the consumer loop share one
// copy, which keeps the kernel's instruction footprint (and instruction-cache
// misses) down.
__device__ __noinline__ PD describe(const DevModel& M, const StepArgs& a, int kind, int l,
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
    case PH_QKV:  // q, k and v rows as one matrix (the engine's packed copy)
      balanced((M.nq + 2 * M.nkv) * M.hd, idx, M.ncta, r0, r1);
      d.p0 = (const char*)L.w_qkv;
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
    kinds[0] = PH_QKV; kinds[1] = PH_ATT; kinds[2] = PH_OUT; kinds[3] = PH_GU; kinds[4] = PH_DOWN;
    return 5;
  }
  kinds[0] = PH_DN_IN; kinds[1] = PH_DN_ST; kinds[2] = PH_OUT; kinds[3] = PH_GU; kinds[4] = PH_DOWN;
  return 5;
}

// ----------------------------------------------------------------------------
// bounded waits and tagged words
// ----------------------------------------------------------------------------
__device__ __forceinline__ void record_error(int* err, int code) { atomicCAS(err, 0, code); }
__device__ __forceinline__ bool aborted(SmemTail* t) { return *(volatile int*)&t->abort_flag != 0; }
__device__ __forceinline__ void set_abort(SmemTail* t) { *(volatile int*)&t->abort_flag = 1; }

// Give up a wait that started at `start`: true (and abort mode) once the CTA
// aborted or the limit passed.
__device__ __forceinline__ bool give_up(SmemTail* t, int* err, uint64_t start,
                                        long long wait_ns) {
  if (aborted(t)) return true;
  if (global_ns() - start > uint64_t(wait_ns)) {
    record_error(err, MK_ERR_TIMEOUT);
    set_abort(t);
    return true;
  }
  return false;
}

// Wait on a ring mbarrier phase; false (and abort mode) when the wait gave up.
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, SmemTail* t,
                                             int* err, long long wait_ns) {
  if (aborted(t)) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t start = global_ns();
  for (int it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31) == 0 && give_up(t, err, start, wait_ns)) return false;
  }
}

__device__ __forceinline__ uint32_t make_tag(uint32_t seq, int phase) {
  return (seq << 8) | uint32_t(phase & 0xFF);
}
__device__ __forceinline__ void ll_put(unsigned long long* p, float v, uint32_t tag) {
  unsigned long long w = (static_cast<unsigned long long>(tag) << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ unsigned long long ll_get(const unsigned long long* p) {
  unsigned long long w;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}

// Consumer threads cooperatively fetch n tagged values into shared memory
// (dst[i] = value of src[i]) once every tag equals `tag`.  Thread tid handles
// i = tid + j*NCT; all its words are in flight at once.  Returns false on
// timeout / abort (per thread; callers agree through named_sync_or).
template <int MAXK>
__device__ __forceinline__ bool ll_gather(float* dst, const unsigned long long* src, int n,
                                          uint32_t tag, SmemTail* t, int* err,
                                          long long wait_ns, int tid) {
  if (aborted(t)) return false;
  unsigned long long w[MAXK];
  uint64_t start = 0;
  for (int it = 0;; ++it) {
#pragma unroll
    for (int j = 0; j < MAXK; ++j) {
      const int i = tid + j * NCT;
      unsigned long long v = static_cast<unsigned long long>(tag) << 32;
      if (i < n) v = ll_get(src + i);
      w[j] = v;
    }
    bool stale = false;
#pragma unroll
    for (int j = 0; j < MAXK; ++j) stale |= uint32_t(w[j] >> 32) != tag;
    if (!stale) break;
    if (it == 0) start = global_ns();
    else if ((it & 7) == 0 && give_up(t, err, start, wait_ns)) return false;
  }
#pragma unroll
  for (int j = 0; j < MAXK; ++j) {
    const int i = tid + j * NCT;
    if (i < n) dst[i] = __uint_as_float(uint32_t(w[j]));
  }
  return true;
}

// One tagged value by one thread.
__device__ __forceinline__ bool ll_wait1(float& out, const unsigned long long* src, uint32_t tag,
                                         SmemTail* t, int* err, long long wait_ns) {
  if (aborted(t)) return false;
  uint64_t start = 0;
  for (int it = 0;; ++it) {
    const unsigned long long w = ll_get(src);
    if (uint32_t(w >> 32) == tag) {
      out = __uint_as_float(uint32_t(w));
      return true;
    }
    if (it == 0) start = global_ns();
    else if ((it & 7) == 0 && give_up(t, err, start, wait_ns)) return false;
  }
}

// Gather several tagged ranges at once (one polling round trip for all):
// segment i copies n values from src to dst (shared memory).
struct LLSeg {
  const unsigned long long* src;
  float* dst;
  int n;
  uint32_t tag;  // the tag every word of this segment must carry
};

template <int MAXK, int NSEG>
__device__ __forceinline__ bool ll_gather_segs(const LLSeg (&sg)[NSEG], SmemTail* t, int* err,
                                               long long wait_ns, int tid) {
  if (aborted(t)) return false;
  const unsigned long long* src[MAXK];
  float* dst[MAXK];
  uint32_t tg[MAXK];
  int total = 0;
#pragma unroll
  for (int q = 0; q < NSEG; ++q) total += sg[q].n;
#pragma unroll
  for (int j = 0; j < MAXK; ++j) {
    int i = tid + j * NCT;
    src[j] = nullptr;
    dst[j] = nullptr;
    tg[j] = 0;
    if (i < total) {
#pragma unroll
      for (int q = 0; q < NSEG; ++q) {
        if (i >= 0 && i < sg[q].n) {
          src[j] = sg[q].src + i;
          dst[j] = sg[q].dst + i;
          tg[j] = sg[q].tag;
        }
        i -= sg[q].n;
      }
    }
  }
  unsigned long long w[MAXK];
  uint64_t start = 0;
  for (int it = 0;; ++it) {
#pragma unroll
    for (int j = 0; j < MAXK; ++j) {
      unsigned long long v = static_cast<unsigned long long>(tg[j]) << 32;
      if (src[j]) v = ll_get(src[j]);
      w[j] = v;
    }
    bool stale = false;
#pragma unroll
    for (int j = 0; j < MAXK; ++j) stale |= uint32_t(w[j] >> 32) != tg[j];
    if (!stale) break;
    if (it == 0) start = global_ns();
    else if ((it & 7) == 0 && give_up(t, err, start, wait_ns)) return false;
  }
#pragma unroll
  for (int j = 0; j < MAXK; ++j)
    if (dst[j]) *dst[j] = __uint_as_float(uint32_t(w[j]));
  return true;
}

// ----------------------------------------------------------------------------
// GEMV helpers (a warp takes four rows at a time).  Lane l owns 16-byte
// weight vectors v*32 + l of a row (8 bf16 each) and the matching 8
// activation floats.
// ----------------------------------------------------------------------------
// Two interleaved accumulation chains over one 16-byte weight vector.
__device__ __forceinline__ void fma8x2(const uint4 w, const float* x, float& a, float& b) {
  a = fmaf(bf_lo(w.x), x[0], a);
  b = fmaf(bf_hi(w.x), x[1], b);
  a = fmaf(bf_lo(w.y), x[2], a);
  b = fmaf(bf_hi(w.y), x[3], b);
  a = fmaf(bf_lo(w.z), x[4], a);
  b = fmaf(bf_hi(w.z), x[5], b);
  a = fmaf(bf_lo(w.w), x[6], a);
  b = fmaf(bf_hi(w.w), x[7], b);
}

// This lane's partial dot products of R rows (in shared memory) with the
// activation (shared memory): lane l takes 16-byte vectors l, l+32, ... of
// each row and the matching 8 activation floats, read once for the R rows.
// One runtime loop serves every row length: the kernel runs each phase's
// code once per token, so a compact instruction footprint beats per-length
// unrolled copies.
template <int R>
__device__ __forceinline__ void dot_rows(const unsigned char* const (&rows)[4], const float* xs,
                                         int nvec, int lane, float (&acc)[R]) {
  const uint4* w[R];
#pragma unroll
  for (int q = 0; q < R; ++q) w[q] = reinterpret_cast<const uint4*>(rows[q]);
  float s[R][2];
#pragma unroll
  for (int q = 0; q < R; ++q) s[q][0] = s[q][1] = 0.f;
  for (int idx = lane; idx < nvec; idx += 32) {
    const float4 p = reinterpret_cast<const float4*>(xs)[idx * 2];
    const float4 h = reinterpret_cast<const float4*>(xs)[idx * 2 + 1];
    const float x[8] = {p.x, p.y, p.z, p.w, h.x, h.y, h.z, h.w};
    uint4 u[R];
#pragma unroll
    for (int q = 0; q < R; ++q) u[q] = w[q][idx];
#pragma unroll
    for (int q = 0; q < R; ++q) fma8x2(u[q], x, s[q][0], s[q][1]);
  }
#pragma unroll
  for (int q = 0; q < R; ++q) acc[q] = s[q][0] + s[q][1];
}

// Warp reduction of two values at once: lanes 0-15 end with the sum of a,
// lanes 16-31 with the sum of b (5 shuffles instead of 10).
__device__ __forceinline__ float reduce2(float a, float b, int lane) {
  const bool h16 = (lane & 16) != 0;
  float x = h16 ? b : a;
  x += __shfl_xor_sync(0xffffffffu, h16 ? a : b, 16);
  x += __shfl_xor_sync(0xffffffffu, x, 8);
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x;
}

// ---- matrix phases ------------------------------------------------------------
// One routine serves every matrix phase, so the hot loop exists once in the
// instruction stream (a phase switch then finds it cached); the epilogue is a
// small runtime switch.
enum EpiKind { EPI_STORE, EPI_RESID, EPI_INPROJ, EPI_SWIGLU, EPI_LOGITS };

struct GemvJob {
  PD d;
  int epi;                   // EpiKind
  unsigned long long* dst;   // tagged destination, indexed by row
  const float* xraw;         // EPI_RESID: residual before the update (shared memory)
  float* hidden;             // EPI_RESID: optional per-layer dump
  const float4* conv_s;      // EPI_INPROJ: conv history rows staged in shared memory
  const uint2* conv_taps;    // EPI_INPROJ: conv taps rows staged in shared memory
  float4* conv_out;          // EPI_INPROJ: the layer's conv history in global memory
  int ch;                    // EPI_INPROJ: conv channels (rows below ch get the conv)
  float* logits;             // EPI_LOGITS
  uint32_t tag;
};

__device__ __forceinline__ void gemv_epilogue(const GemvJob& j, int row, float y, float y2,
                                              float& best_v, int& best_i) {
  switch (j.epi) {
    case EPI_STORE:
      ll_put(j.dst + row, y, j.tag);
      break;
    case EPI_RESID: {
      const float v = j.xraw[row] + y;
      ll_put(j.dst + row, v, j.tag);
      if (j.hidden) j.hidden[row] = v;
      break;
    }
    case EPI_INPROJ:
      if (row < j.ch) {
        // taps (u_{t-3}, u_{t-2}, u_{t-1}, u_t); shift the history by one
        const float4 s = j.conv_s[row - j.d.r0];
        const uint2 wc = j.conv_taps[row - j.d.r0];
        const float c =
            bf_lo(wc.x) * s.x + bf_hi(wc.x) * s.y + bf_lo(wc.y) * s.z + bf_hi(wc.y) * y;
        j.conv_out[row] = make_float4(s.y, s.z, y, 0.f);
        ll_put(j.dst + row, siluf_(c), j.tag);
      } else {
        ll_put(j.dst + row, y, j.tag);
      }
      break;
    case EPI_SWIGLU:
      ll_put(j.dst + row, siluf_(y) * y2, j.tag);
      break;
    case EPI_LOGITS:
      j.logits[row] = y;
      if (y > best_v || (y == best_v && row < best_i)) {
        best_v = y;
        best_i = row;
      }
      break;
  }
}

// Walk the CTA's chunks of one matrix phase.  Each warp takes its rows of a
// chunk up to four at a time (rows i, i+NCW, i+2NCW, i+3NCW; for EPI_SWIGLU
// the gate and up rows of i and i+NCW), computes only the dot products of
// rows that exist, reduces them in one transposed shuffle tree and parks
// each result in lane (count of results so far); the epilogue then runs once
// per 32 results with every lane finishing its own row, instead of one lane
// finishing rows one by one.
// The activation vector is in shared memory (xs).  Returns the chunk counter
// after the phase.
__device__ __forceinline__ uint32_t gemv_core(const GemvJob& j, uint32_t g, unsigned char* ring,
                                              SmemTail* t, int* err, long long wait_ns,
                                              const float* xs) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PD& d = j.d;
  const int nvec = int(d.row_bytes / 16);
  const bool swiglu = j.epi == EPI_SWIGLU;
  float best_v = -INFINITY;
  int best_i = 0x7FFFFFFF;
  float kv = 0.f, kv2 = 0.f;  // parked result (and up value for EPI_SWIGLU) of this lane
  int krow = 0, nb = 0;       // its row; number of parked results in the warp
  int local = 0;
#pragma unroll 1
  for (int r = d.r0; r < d.r0 + d.n; r += d.rpc, ++g, local += d.rpc) {
    const int slot = int(g % NSLOT);
    if (bounded_wait(&t->full[slot], (g / NSLOT) & 1, t, err, wait_ns)) {
      const int nr = min(d.rpc, d.r0 + d.n - r);
      const unsigned char* base = ring + size_t(slot) * SLOT;
      const size_t rb = d.row_bytes;
      const int step = swiglu ? 2 * NCW : 4 * NCW;
#pragma unroll 1
      for (int i = (warp - (local % NCW) + NCW) % NCW; i < nr; i += step) {
        int nout;
        const unsigned char *p0, *p1, *p2, *p3;
        if (swiglu) {
          nout = i + NCW < nr ? 2 : 1;
          const int i1 = nout > 1 ? i + NCW : i;
          p0 = base + size_t(i) * rb;
          p1 = base + size_t(d.rpc + i) * rb;
          p2 = base + size_t(i1) * rb;
          p3 = base + size_t(d.rpc + i1) * rb;
        } else {
          nout = min(4, (nr - i + NCW - 1) / NCW);
          p0 = base + size_t(i) * rb;
          p1 = base + size_t(nout > 1 ? i + NCW : i) * rb;
          p2 = base + size_t(nout > 2 ? i + 2 * NCW : i) * rb;
          p3 = base + size_t(nout > 3 ? i + 3 * NCW : i) * rb;
        }
        // as many row dot products as this iteration has rows (a slot holds
        // few rows per warp, so most iterations have one or two)
        const unsigned char* const rows[4] = {p0, p1, p2, p3};
        const int R = swiglu ? 2 * nout : (nout == 3 ? 4 : nout);
        float z;
        int sh;  // result q of the reduction sits in lanes q << sh ...
        if (R == 1) {
          float a1[1];
          dot_rows<1>(rows, xs, nvec, lane, a1);
          z = warp_sum(a1[0]);
          sh = 5;
        } else if (R == 2) {
          float a2[2];
          dot_rows<2>(rows, xs, nvec, lane, a2);
          z = reduce2(a2[0], a2[1], lane);
          sh = 4;
        } else {
          float a4[4];
          dot_rows<4>(rows, xs, nvec, lane, a4);
          z = reduce4(a4[0], a4[1], a4[2], a4[3], lane);
          sh = 3;
        }
        if (nb + nout > 32) {
          if (lane < nb) gemv_epilogue(j, krow, kv, kv2, best_v, best_i);
          nb = 0;
        }
        const int q = lane - nb;
        if (swiglu) {  // results 2o (gate) and 2o+1 (up) of output o
          const float gv = __shfl_sync(0xffffffffu, z, (2 * (q & 1)) << sh);
          const float uv = __shfl_sync(0xffffffffu, z, (2 * (q & 1) + 1) << sh);
          if (q >= 0 && q < nout) {
            kv = gv;
            kv2 = uv;
            krow = r + i + q * NCW;
          }
        } else {
          const float v = __shfl_sync(0xffffffffu, z, (q & (R - 1)) << sh);
          if (q >= 0 && q < nout) {
            kv = v;
            krow = r + i + q * NCW;
          }
        }
        nb += nout;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&t->empty[slot]);
  }
  if (lane < nb) gemv_epilogue(j, krow, kv, kv2, best_v, best_i);
  if (j.epi == EPI_LOGITS && best_i != 0x7FFFFFFF)
    atomicMax(&t->best, pack_argmax(best_v, best_i));
  return g;
}

// ----------------------------------------------------------------------------
// RMSNorm of the vector already in `xin` (all NCT consumer threads):
// xin = xin * rsqrt(mean(xin^2) + eps) * gain, keeping the raw copy in xraw.
// ----------------------------------------------------------------------------
// Gains of RMSNorm as this thread uses them (element tid + k*NCT), loaded
// before the input is awaited so their latency overlaps the wait.
constexpr int GK = per_thread(XRAW_MAX);
__device__ __forceinline__ void load_gains(float (&gv)[GK], const uint16_t* gain, int H, int tid) {
#pragma unroll
  for (int k = 0; k < GK; ++k) {
    const int i = tid + k * NCT;
    gv[k] = (gain && i < H) ? bf2f(gain[i]) : 1.f;
  }
}

__device__ __forceinline__ void rmsnorm_inplace(float* xin, float* xraw, const float (&gv)[GK],
                                                int H, float eps, SmemTail* t, int tid) {
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < GK; ++k) {
    const int i = tid + k * NCT;
    if (i < H) {
      const float v = xin[i];
      if (xraw) xraw[i] = v;
      ss = fmaf(v, v, ss);
    }
  }
  ss = warp_sum(ss);
  if ((tid & 31) == 0) t->red[tid >> 5] = ss;
  named_sync(1, NCT);
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < NCW; ++w) tot += t->red[w];
  const float inv = 1.0f / sqrtf(tot / float(H) + eps);
#pragma unroll
  for (int k = 0; k < GK; ++k) {
    const int i = tid + k * NCT;
    if (i < H) xin[i] = xin[i] * inv * gv[k];
  }
  named_sync(1, NCT);
}

// Chunk loop for the non-GEMV phases (state rows, KV positions): the body
// sees `row`, `p0` (plane-0 row in shared memory) and `p1` (plane-1 row).
// (A macro: the body must be inlined so register arrays stay in registers.)
#define MK_CHUNK_LOOP(d, ...)                                                          \
  do {                                                                                 \
    int local_ = 0;                                                                    \
    for (int r_ = (d).r0; r_ < (d).r0 + (d).n; r_ += (d).rpc, ++g, local_ += (d).rpc) { \
      const int slot_ = int(g % NSLOT);                                                \
      const bool ok_ = bounded_wait(&t->full[slot_], (g / NSLOT) & 1, t, M.err, a.wait_ns); \
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
                                               uint32_t tag_in, uint32_t tag_out, bool dry,
                                               int tid, int warp, int lane) {
  constexpr int EPL = DK / 32;
  constexpr int stride = 2 * DK + 4;  // head cache: [q(dk) | k(dk) | beta, alpha, k.q, -]
  const int h_first = d.n > 0 ? d.r0 / M.dv : 0;
  const int n_heads = d.n > 0 ? (d.r0 + d.n - 1) / M.dv - h_first + 1 : 0;
  // staging: raw q, k of the touched heads, v of this CTA's rows, b and a
  float* sq_raw = uni + DN_HEADS_MAX * stride;   // [n_heads][DK]
  float* sk_raw = sq_raw + DN_HEADS_MAX * DK;    // [n_heads][DK]
  float* vrow = sk_raw + DN_HEADS_MAX * DK;      // [d.n]
  float* sba = vrow + DN_ROWS_MAX;               // [2][n_heads]
  bool ok = true;
  if (!dry && d.n > 0) {
    const LLSeg sg[5] = {
        {M.inp_ll + h_first * DK, sq_raw, n_heads * DK, tag_in},
        {M.inp_ll + M.nh * DK + h_first * DK, sk_raw, n_heads * DK, tag_in},
        {M.inp_ll + 2 * M.nh * DK + d.r0, vrow, d.n, tag_in},
        {M.inp_ll + M.ch + M.nh * M.dv + h_first, sba, n_heads, tag_in},
        {M.inp_ll + M.ch + M.nh * M.dv + M.nh + h_first, sba + DN_HEADS_MAX, n_heads, tag_in}};
    ok = ll_gather_segs<per_thread(2 * DN_HEADS_MAX * DK + DN_ROWS_MAX + 2 * DN_HEADS_MAX), 5>(
        sg, t, M.err, a.wait_ns, tid);
  }
  const bool bad = named_sync_or(1, NCT, !ok);
  if (!dry && !bad) {
    for (int hh = warp; hh < n_heads; hh += NCW) {
      const int h = h_first + hh;
      float qv[EPL], kv[EPL];
      float sq = 0.f, sk = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        qv[e] = sq_raw[hh * DK + lane * EPL + e];
        kv[e] = sk_raw[hh * DK + lane * EPL + e];
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
        const float b = sba[hh], aa = sba[DN_HEADS_MAX + hh];
        uni[hh * stride + 2 * DK + 0] = sigmoidf_(b);  // beta
        uni[hh * stride + 2 * DK + 1] =
            expf(-expf(L.A_log[h]) * softplusf_(aa + L.dt_bias[h]));  // alpha
        uni[hh * stride + 2 * DK + 2] = kq;
      }
    }
  }
  named_sync(1, NCT);
  float* st = M.dn_state[a.st_buf] + size_t(L.sub) * M.nh * M.dv * DK;
  MK_CHUNK_LOOP(d, {
    const int h = row / M.dv;
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
    const float u = beta * (vrow[row - d.r0] - alpha * s_k);  // S' = alpha S + u k^T
    float* dst = st + size_t(row) * DK + lane * EPL;
    if constexpr (EPL == 4) {
      *reinterpret_cast<float4*>(dst) =
          make_float4(fmaf(alpha, sv[0], u * kv[0]), fmaf(alpha, sv[1], u * kv[1]),
                      fmaf(alpha, sv[2], u * kv[2]), fmaf(alpha, sv[3], u * kv[3]));
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) dst[e] = fmaf(alpha, sv[e], u * kv[e]);
    }
    if (lane == 0) ll_put(M.dno_ll + row, fmaf(alpha, s_q, u * kq), tag_out);  // o_i = S'_i.q
  });
}

// One key/value row into a warp's online-softmax state for G query heads
// (this lane's EPL elements of the row).
template <int G, int EPL>
__device__ __forceinline__ void att_consume(float (&am)[G], float (&al)[G], float (&acc)[G][EPL],
                                            const float (&qr)[G][EPL], const float* kf,
                                            const float* vf, float scale) {
  float sc[G];
  if constexpr (G == 4) {
    // the four heads' scores reduced together, then broadcast from lane 8j
    float pz[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      pz[j] = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) pz[j] = fmaf(qr[j][e], kf[e], pz[j]);
    }
    const float z = reduce4(pz[0], pz[1], pz[2], pz[3], threadIdx.x & 31);
#pragma unroll
    for (int j = 0; j < 4; ++j) sc[j] = __shfl_sync(0xffffffffu, z, 8 * j) * scale;
  } else {
#pragma unroll
    for (int j = 0; j < G; ++j) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) s = fmaf(qr[j][e], kf[e], s);
      sc[j] = warp_sum(s) * scale;
    }
  }
#pragma unroll
  for (int j = 0; j < G; ++j) {
    const float mn = fmaxf(am[j], sc[j]);
    const float corr = expf(am[j] - mn);
    const float pr = expf(sc[j] - mn);
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
                                                uint32_t tag_qkv, uint32_t tag_dbg,
                                                uint32_t tag_out, bool dry, int tid, int warp,
                                                int lane) {
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
  const int half = HD / 2;
  bool ok = true;
  if (unit && !dry) {
    // raw q of the group's heads (staged in att_acc) and, for the split that
    // owns the new position, its raw k and v: one polling round
    const LLSeg sg[3] = {
        {M.qkv_ll + gidx * G * HD, att_acc, G * HD, tag_qkv | tag_dbg},
        {M.qkv_ll + M.nq * HD + gidx * HD, att_kn, last ? HD : 0, tag_qkv},
        {M.qkv_ll + (M.nq + M.nkv) * HD + gidx * HD, att_vn, last ? HD : 0, tag_qkv}};
    ok = ll_gather_segs<per_thread(GQ * HD + 2 * HD), 3>(sg, t, M.err, a.wait_ns, tid);
  }
  const bool bad = named_sync_or(1, NCT, !ok);
  const bool work = unit && !dry && !bad;
  if (work) {
    for (int i = tid; i < G * half; i += NCT) {
      const int j = i / half, c = i % half;
      const float x0 = att_acc[j * HD + c], x1 = att_acc[j * HD + c + half];
      const float cs = t->rope_cos[c], sn = t->rope_sin[c];
      att_q[j * HD + c] = x0 * cs - x1 * sn;
      att_q[j * HD + c + half] = x1 * cs + x0 * sn;
    }
  }
  named_sync(1, NCT);
  if (work) {
    for (int i = tid; i < G * HD; i += NCT) att_acc[i] = 0.f;
    if (last) {
      // RoPE the new key, store K/V at `pos` in bf16, keep the rounded values
      const size_t cofs = ((size_t(L.sub) * M.nkv + gidx) * M.max_ctx + a.pos) * HD;
      for (int c = tid; c < half; c += NCT) {
        const float x0 = att_kn[c], x1 = att_kn[c + half];
        const float cs = t->rope_cos[c], sn = t->rope_sin[c];
        const uint16_t b0 = f2bf(x0 * cs - x1 * sn), b1 = f2bf(x1 * cs + x0 * sn);
        M.kc[cofs + c] = b0;
        M.kc[cofs + c + half] = b1;
        att_kn[c] = bf2f(b0);
        att_kn[c + half] = bf2f(b1);
      }
      for (int c = tid; c < HD; c += NCT) {
        const uint16_t b = f2bf(att_vn[c]);
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
      qr[j][e] = att_q[j * HD + lane * EPL + e];
    }
  }
  const float scale = 1.0f / sqrtf(float(HD));
  MK_CHUNK_LOOP(d, {
    const uint16_t* k16 = reinterpret_cast<const uint16_t*>(p0) + lane * EPL;
    const uint16_t* v16 = reinterpret_cast<const uint16_t*>(p1) + lane * EPL;
    float kf[EPL], vf[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      kf[e] = bf2f(k16[e]);
      vf[e] = bf2f(v16[e]);
    }
    att_consume<G, EPL>(am, al, acc, qr, kf, vf, scale);
  });
  const bool dry_post = named_sync_or(1, NCT, aborted(t) || !work);
  if (dry_post) return;
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
  // publish this split's partial as tagged words: per head [acc(HD) | m | l]
  unsigned long long* part = M.part_ll + size_t(gidx) * kMaxCtas * G * (HD + 2);
  unsigned long long* pbase = part + size_t(d.unit_s) * G * (HD + 2);
  for (int i = tid; i < G * HD; i += NCT) ll_put(pbase + (i / HD) * (HD + 2) + (i % HD), att_acc[i], tag_out);
  if (tid < G) {
    float mx = -INFINITY, ls = 0.f;
    for (int w = 0; w < NCW; ++w) mx = fmaxf(mx, att_ml[(w * G + tid) * 2]);
    for (int w = 0; w < NCW; ++w) {
      const float lw = att_ml[(w * G + tid) * 2 + 1];
      if (lw > 0.f) ls += lw * expf(att_ml[(w * G + tid) * 2] - mx);
    }
    ll_put(pbase + tid * (HD + 2) + HD, mx, tag_out);
    ll_put(pbase + tid * (HD + 2) + HD + 1, ls, tag_out);
  }
  // Cooperative merge: every split CTA of the group merges its slice
  // [e0, e1) of the group's G*HD outputs from all S partials.  The (m, l)
  // words of all splits double as the group's completion signal.
  const int S = d.S;
  const int e0 = (G * HD) * d.unit_s / S, e1 = (G * HD) * (d.unit_s + 1) / S;
  const int ne = e1 - e0;
  constexpr int ATT_SCRATCH = 2 * G * HD + 2 * HD + NCW * G * 2;
  float* mls = uni + ATT_SCRATCH;  // [S][G][2]  (m, l) of every split
  float* wgt = mls + S * G * 2;    // [S][G]     merge weights
  float* stage = uni;              // [S][ne]    the slice's partial values (att_q is free now)
  bool ok2 = true;
  {
    uint64_t start = 0;
    for (int it = 0;; ++it) {
      bool stale = false;
#pragma unroll 4
      for (int w = tid; w < S * G * 2; w += NCT) {
        const int si = w / (G * 2), j = (w >> 1) % G, c = w & 1;
        const unsigned long long v = ll_get(part + (size_t(si) * G + j) * (HD + 2) + HD + c);
        if (uint32_t(v >> 32) != tag_out) stale = true;
        else mls[w] = __uint_as_float(uint32_t(v));
      }
      if (!stale) break;
      if (it == 0) start = global_ns();
      else if ((it & 7) == 0 && give_up(t, M.err, start, a.wait_ns)) { ok2 = false; break; }
    }
  }
  if (named_sync_or(1, NCT, !ok2)) return;
  if (tid < G) {
    float mx = -INFINITY;
    for (int si = 0; si < S; ++si) mx = fmaxf(mx, mls[(si * G + tid) * 2]);
    float den = 0.f;
    for (int si = 0; si < S; ++si) {
      const float f = expf(mls[(si * G + tid) * 2] - mx);
      wgt[si * G + tid] = f;
      den = fmaf(f, mls[(si * G + tid) * 2 + 1], den);
    }
    const float inv = 1.0f / den;
    for (int si = 0; si < S; ++si) wgt[si * G + tid] *= inv;
  }
  {
    uint64_t start = 0;
    for (int it = 0;; ++it) {
      bool stale = false;
#pragma unroll 4
      for (int w = tid; w < S * ne; w += NCT) {
        const int si = w / ne, e = e0 + w % ne;
        const unsigned long long v = ll_get(part + (size_t(si) * G + e / HD) * (HD + 2) + e % HD);
        if (uint32_t(v >> 32) != tag_out) stale = true;
        else stage[w] = __uint_as_float(uint32_t(v));
      }
      if (!stale) break;
      if (it == 0) start = global_ns();
      else if ((it & 7) == 0 && give_up(t, M.err, start, a.wait_ns)) { ok2 = false; break; }
    }
  }
  if (named_sync_or(1, NCT, !ok2)) return;
  for (int w = tid; w < ne; w += NCT) {
    const int e = e0 + w, j = e / HD;
    float o = 0.f;
    for (int si = 0; si < S; ++si) o = fmaf(wgt[si * G + j], stage[si * ne + w], o);
    ll_put(M.atto_ll + size_t(gidx) * G * HD + e, o, tag_out);
  }
}

// ----------------------------------------------------------------------------
// Cursor over one CTA's chunk schedule for one launch: every phase of every
// layer, then the LM head, each split into chunks of at most `rpc` rows.
// ----------------------------------------------------------------------------
constexpr size_t PF_AHEAD = size_t(64) << 10;  // L2 prefetch distance per CTA (bytes)

struct ChunkCursor {
  int l, p, np, gp;
  int kinds[8];
  PD d;
  int r;      // first row of the current chunk
  bool done;
  __device__ __forceinline__ int nrows() const { return min(d.rpc, d.r0 + d.n - r); }
  __device__ __forceinline__ uint32_t bytes() const { return uint32_t(nrows()) * d.row_bytes; }
  __device__ __forceinline__ const char* src0() const { return d.p0 + size_t(r) * d.row_bytes; }
  __device__ __forceinline__ const char* src1() const { return d.p1 + size_t(r) * d.row_bytes; }
};

// Move to the first chunk at or after phase (l, p); skips empty phases.
__device__ __noinline__ void cursor_settle(ChunkCursor& c, const DevModel& M,
                                              const StepArgs& a, int cta, uint64_t pol_w,
                                              uint64_t pol_s) {
  while (true) {
    if (c.l > M.n_layers) {
      c.done = true;
      return;
    }
    if (c.p >= c.np) {
      ++c.l;
      c.p = 0;
      if (c.l < M.n_layers) c.np = layer_phases(M.layers[c.l], c.kinds);
      else if (c.l == M.n_layers) { c.kinds[0] = PH_LM; c.np = 1; }
      continue;
    }
    c.d = describe(M, a, c.kinds[c.p], c.l < M.n_layers ? c.l : 0, c.gp, cta, pol_w, pol_s);
    c.r = c.d.r0;
    if (c.d.n > 0) return;
    ++c.p;
    ++c.gp;
  }
}

__device__ __forceinline__ void cursor_init(ChunkCursor& c, const DevModel& M, const StepArgs& a,
                                            int cta, uint64_t pol_w, uint64_t pol_s) {
  c.l = 0;
  c.p = 0;
  c.gp = 0;
  c.done = false;
  c.np = layer_phases(M.layers[0], c.kinds);
  cursor_settle(c, M, a, cta, pol_w, pol_s);
}

__device__ __forceinline__ void cursor_next(ChunkCursor& c, const DevModel& M, const StepArgs& a,
                                            int cta, uint64_t pol_w, uint64_t pol_s) {
  c.r += c.d.rpc;
  if (c.r < c.d.r0 + c.d.n) return;
  ++c.p;
  ++c.gp;
  cursor_settle(c, M, a, cta, pol_w, pol_s);
}

// ----------------------------------------------------------------------------
// the kernel
// ----------------------------------------------------------------------------
template <int DK, int HD, int GQ>
__global__ void __launch_bounds__(NTHR, 1) decode_kernel(const __grid_constant__ StepArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* ring = smem_raw;
  SmemTail* t = reinterpret_cast<SmemTail*>(smem_raw + size_t(NSLOT) * SLOT);
  float* uni = reinterpret_cast<float*>(smem_raw + size_t(NSLOT) * SLOT + sizeof(SmemTail));
  float* xraw = uni + UNION_FLOATS;

  const DevModel& M = a.m;
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
  // Two cursors walk the same chunk schedule: the load cursor fills the
  // shared-memory ring (TMA bulk copies, waits for free slots); the prefetch
  // cursor runs up to PF_AHEAD bytes ahead issuing L2 bulk prefetches, so HBM
  // keeps streaming while the consumers wait for other CTAs and the ring
  // refills from L2.
  if (warp == NCW) {
    if (lane != 0) return;
    ChunkCursor ld, pf;
    cursor_init(ld, M, a, cta, pol_w, pol_s);
    cursor_init(pf, M, a, cta, pol_w, pol_s);
    size_t ld_bytes = 0, pf_bytes = 0;
    uint32_t g = 0;
    while (!ld.done && !aborted(t)) {
      // keep the prefetch cursor PF_AHEAD bytes ahead of the loads
      while (!pf.done && pf_bytes < ld_bytes + PF_AHEAD) {
        const uint32_t b = pf.bytes();
        bulk_prefetch_l2(pf.src0(), b);
        if (pf.d.p1) bulk_prefetch_l2(pf.src1(), b);
        pf_bytes += size_t(b) * (pf.d.p1 ? 2 : 1);
        cursor_next(pf, M, a, cta, pol_w, pol_s);
      }
      const int slot = int(g % NSLOT);
      if (g >= NSLOT && !bounded_wait(&t->empty[slot], ((g / NSLOT) - 1) & 1, t, M.err, a.wait_ns))
        break;
      const uint32_t bytes = ld.bytes();
      unsigned char* dst = ring + size_t(slot) * SLOT;
      mbar_arrive_expect_tx(&t->full[slot], bytes * (ld.d.p1 ? 2u : 1u));
      bulk_g2s(dst, ld.src0(), bytes, &t->full[slot], ld.d.pol);
      if (ld.d.p1)
        bulk_g2s(dst + size_t(ld.d.rpc) * ld.d.row_bytes, ld.src1(), bytes, &t->full[slot], ld.d.pol);
      ld_bytes += size_t(bytes) * (ld.d.p1 ? 2 : 1);
      ++g;
      cursor_next(ld, M, a, cta, pol_w, pol_s);
    }
    // Let every copy still in flight land before the CTA may exit.
    const uint32_t first = g > uint32_t(NSLOT) ? g - NSLOT : 0u;
    for (uint32_t q = first; q < g; ++q) {
      const uint64_t start = global_ns();
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
  int gp = 0;
  int kinds[8];
  // tags of the latest producer of each tagged buffer
  uint32_t tag_x = 0, tag_inp = 0, tag_dno = 0, tag_qkv = 0, tag_att = 0,
           tag_h = 0;
  int xb = 0;  // residual buffer holding the latest x

  for (int l = 0; l <= M.n_layers; ++l) {
    const bool lm = (l == M.n_layers);
    const DevLayer& L = M.layers[lm ? 0 : l];
    int np;
    if (!lm) np = layer_phases(L, kinds);
    else { kinds[0] = PH_LM; np = 1; }

    for (int p = 0; p < np; ++p, ++gp) {
      const int kind = kinds[p];
      const PD d = describe(M, a, kind, lm ? 0 : l, gp, cta, pol_w, pol_s);
      const uint32_t tag_me = make_tag(a.seq, gp);
      // debug hook: the inputs of phase `fail_phase` carry a tag nobody writes
      const uint32_t dbg = gp == a.fail_phase ? 0x80000000u : 0u;
      // uniform across the consumer warps (also orders the previous phase)
      const bool dry = named_sync_or(1, NCT, aborted(t));
      GemvJob j{};  // matrix phases fill it in; one dispatch after the switch
      j.d = d;
      j.tag = tag_me;
      bool gemv = false;
      switch (kind) {
        case PH_DN_IN:
        case PH_QKV:
        case PH_GU:
        case PH_LM: {
          // input: RMSNorm of the residual stream (the embedding at layer 0)
          bool ok = true;
          // union layout in this phase: x [0, 2048) | conv history [2048, 3072)
          // (<= CONV_ROWS_MAX float4) | conv taps [3072, 3584) (<= CONV_ROWS_MAX uint2)
          float4* conv_s = reinterpret_cast<float4*>(uni + 2048);
          uint2* conv_taps = reinterpret_cast<uint2*>(uni + 2048 + 4 * CONV_ROWS_MAX);
          float4* conv_g = reinterpret_cast<float4*>(M.conv_state[a.st_buf]) + size_t(L.sub) * M.ch;
          const uint16_t* gain = kind == PH_GU ? L.mlp_norm
                                 : kind == PH_LM ? M.final_norm : L.attn_norm;
          float gv[GK];
          load_gains(gv, gain, M.H, tid);
          if (!dry) {
            if (kind == PH_DN_IN) {
              // stage the conv history and taps of this CTA's q|k|v rows first
              // (independent of the input: their latency overlaps the wait)
              const int nconv = max(0, min(d.r0 + d.n, M.ch) - d.r0);
              for (int i = tid; i < nconv; i += NCT) {
                conv_s[i] = conv_g[d.r0 + i];
                conv_taps[i] = *reinterpret_cast<const uint2*>(L.conv_w + size_t(d.r0 + i) * 4);
              }
            }
            if (l == 0 && kind != PH_GU) {
              for (int i = tid; i < M.H; i += NCT) uni[i] = bf2f(emb_row[i]);
            } else {
              ok = ll_gather<per_thread(XRAW_MAX)>(uni, M.x_ll + size_t(xb) * M.H, M.H,
                                                   tag_x | dbg, t, M.err, a.wait_ns, tid);
            }
          }
          const bool bad = named_sync_or(1, NCT, !ok);
          if (!dry && !bad)
            rmsnorm_inplace(uni, kind == PH_LM ? nullptr : xraw, gv, M.H, M.eps, t, tid);
          gemv = true;
          if (kind == PH_DN_IN) {
            j.epi = EPI_INPROJ;
            j.dst = M.inp_ll;
            j.conv_s = conv_s;
            j.conv_taps = conv_taps;
            j.conv_out = conv_g;
            j.ch = M.ch;
            tag_inp = tag_me;
          } else if (kind == PH_QKV) {
            j.epi = EPI_STORE;
            j.dst = M.qkv_ll;  // [q | k | v], the rows' order
            tag_qkv = tag_me;
          } else if (kind == PH_GU) {
            j.epi = EPI_SWIGLU;
            j.dst = M.mlph_ll;
            tag_h = tag_me;
          } else {
            j.epi = EPI_LOGITS;
            j.logits = a.logits;
          }
          break;
        }
        case PH_OUT: {
          bool ok = true;
          const int K = L.is_attn ? M.nq * M.hd : M.nh * M.dv;
          constexpr int EPL_G = DK / 32;  // gated-norm elements per lane (dv == dk)
          float gw[EPL_G];
#pragma unroll
          for (int e = 0; e < EPL_G; ++e) gw[e] = L.is_attn ? 0.f : bf2f(L.out_norm[lane * EPL_G + e]);
          if (!dry) {
            if (L.is_attn) {
              ok = ll_gather<per_thread(UNION_FLOATS)>(uni, M.atto_ll, K, tag_att | dbg, t, M.err,
                                                       a.wait_ns, tid);
            } else {
              // gated RMSNorm of the readout: o_h from the state phase, z_h
              // from the in-projection (z staged in the upper half of uni)
              // o (tagged by the state phase) and z (by the in-projection)
              // in one polling round
              const LLSeg sg[2] = {{M.dno_ll, uni, K, tag_dno | dbg},
                                   {M.inp_ll + M.ch, uni + 2048, K, tag_inp}};
              ok = ll_gather_segs<per_thread(4096), 2>(sg, t, M.err, a.wait_ns, tid);
            }
          }
          const bool bad = named_sync_or(1, NCT, !ok);
          if (!dry && !bad && !L.is_attn) {
            constexpr int EPL = DK / 32;  // dv == dk
            for (int h = warp; h < M.nh; h += NCW) {
              float o[EPL];
              float ss = 0.f;
#pragma unroll
              for (int e = 0; e < EPL; ++e) {
                o[e] = uni[h * DK + lane * EPL + e];
                ss = fmaf(o[e], o[e], ss);
              }
              ss = warp_sum(ss);
              const float inv = 1.0f / sqrtf(ss / float(DK) + M.eps);
#pragma unroll
              for (int e = 0; e < EPL; ++e) {
                const int i = lane * EPL + e;
                uni[h * DK + i] = o[e] * inv * gw[e] * siluf_(uni[2048 + h * DK + i]);
              }
            }
            named_sync(1, NCT);
          }
          gemv = true;
          j.epi = EPI_RESID;
          j.dst = M.x_ll + size_t(xb ^ 1) * M.H;
          j.xraw = xraw;
          xb ^= 1;
          tag_x = tag_me;
          break;
        }
        case PH_DOWN: {
          bool ok = true;
          if (!dry)
            ok = ll_gather<per_thread(UNION_FLOATS)>(uni, M.mlph_ll, M.I, tag_h | dbg, t, M.err,
                                                     a.wait_ns, tid);
          named_sync_or(1, NCT, !ok);
          gemv = true;
          j.epi = EPI_RESID;
          j.dst = M.x_ll + size_t(xb ^ 1) * M.H;
          j.xraw = xraw;
          j.hidden = a.hidden ? a.hidden + size_t(l) * M.H : nullptr;
          xb ^= 1;
          tag_x = tag_me;
          break;
        }
        case PH_DN_ST:
          dn_state_phase<DK>(M, a, L, d, g, ring, t, uni, tag_inp | dbg, tag_me, dry, tid, warp,
                             lane);
          tag_dno = tag_me;
          break;
        case PH_ATT:
          attention_phase<HD, GQ>(M, a, L, d, g, ring, t, uni, tag_qkv, dbg, tag_me,
                                  dry, tid, warp, lane);
          tag_att = tag_me;
          break;
        default:
          break;
      }
      if (gemv) g = gemv_core(j, g, ring, t, M.err, a.wait_ns, uni);
    }
  }

  // ---------------- argmax over the grid ----------------
  const bool bad = named_sync_or(1, NCT, aborted(t));
  if (tid == 0 && !bad) {
    if (t->best) atomicMax(&M.amax[a.amax_out], t->best);
    __threadfence();
    unsigned* tk = M.tickets;
    const unsigned prev = atomicAdd(tk, 1u);
    if (prev == unsigned(M.ncta - 1)) {
      atomicExch(tk, 0u);
      __threadfence();
      const unsigned long long v = atomicAdd(&M.amax[a.amax_out], 0ull);
      if (a.tok_out) *a.tok_out = int(0xFFFFFFFFu - uint32_t(v & 0xFFFFFFFFull));
      // every CTA has read its input token by now: clear the slot the next
      // launch accumulates into
      M.amax[a.amax_in] = 0ull;
    }
  }
}

}  // namespace mk
