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
//  * The grid is split into ng groups of gs CTAs, one group per DeltaNet
//    head (the 0.8B-shaped model: 16 groups of 9 CTAs; leftover SMs join
//    the phases that are split over the whole grid).  A group computes its
//    head's in-projection rows, exchanges them inside the group, and then
//    every CTA of the group advances the head's whole recurrent state, so
//    the readout and the gated norm need no further exchange.  Projections
//    back to the residual stream (DeltaNet and attention output, MLP down)
//    run split-K: group g owns K block g, its CTAs split the output rows,
//    and the ng partial sums of each output meet in one 64-bit word per
//    output (see "count-carrying sums" below).  The MLP's gate/up rows of
//    K block g are computed inside group g and exchanged inside it.
//  * Each CTA knows its share of every phase at launch, so one producer warp
//    walks the CTA's whole per-token byte stream and keeps a 3 x 64 KB
//    shared-memory ring full with bulk TMA copies (cp.async.bulk + mbarrier
//    complete_tx).  It never waits for other CTAs.
//  * Exchanges carry their own completion: a tagged word {fp32 value,
//    32-bit tag naming launch and phase} for gathers, and for the split-K
//    sums a word {8-bit count | 56-bit biased fixed-point sum} that every
//    contributor adds to with one 64-bit atomic.  Integer addition makes the
//    sum independent of arrival order (bit-reproducible), and a reader knows
//    the sum is complete when the count equals the number of contributors.
//    There is no grid barrier, no fence and no counter on the data path.
//  * Eleven consumer warps: bf16 GEMV rows against fp32 activations in
//    shared memory, the gated delta-rule row update, split-K flash-decode
//    attention with an online softmax, SwiGLU, the tied LM head with a grid
//    argmax.
//  * Every wait is bounded by %globaltimer; on expiry the kernel records
//    MK_ERR_TIMEOUT, runs the rest of its schedule without work, lets its
//    in-flight copies land and returns.
#pragma once
#include "mk_model.cuh"
#include "mk_ptx.cuh"

namespace mk {

constexpr int NCW = 11;                 // consumer warps (12 warps per CTA)
constexpr int NCT = NCW * 32;           // consumer threads
constexpr int NTHR = NCT + 32;          // + producer warp
constexpr int SLOT = 65536;             // ring slot bytes
constexpr int NSLOT = 3;                // ring slots
constexpr int ATT_MIN_POS = 32;         // fewest positions per attention split
constexpr int XRAW_MAX = 2048;          // largest hidden size (residual copy in shared memory)
constexpr int UNION_FLOATS = 4096;      // activation vector | head cache | attention scratch
constexpr int CONV_ROWS_MAX = 256;      // in-projection rows of one CTA (conv staging)
constexpr int MERGE_STAGE = 2048;       // partial values staged per attention-merge batch
constexpr int MERGE_HEADS_MAX = 8;      // q heads one K block of the attention output spans
constexpr int MERGE_ML_MAX = 1200;      // (m, l) words of all splits of those heads

// count-carrying fixed-point sums: word = count << 56 | sum of (round(y * 2^32) + 2^46)
constexpr int CFA_SHIFT = 56;
constexpr unsigned long long CFA_MASK = (1ull << CFA_SHIFT) - 1;
constexpr long long CFA_BIAS = 1ll << 46;
constexpr double CFA_SCALE = 4294967296.0;  // 2^32
constexpr float CFA_LIMIT = 8192.f;         // |contribution| < 2^13 keeps every sum in 56 bits

// words per consumer thread when NCT threads gather n tagged values
constexpr int per_thread(int n) { return (n + NCT - 1) / NCT; }

enum PhaseKind {
  PH_DN_IN,     // DeltaNet in-projection rows of the group's head (+ causal conv)
  PH_DN_ST,     // the head's gated delta rule, readout and gated RMSNorm (whole head per CTA)
  PH_DN_OUTP,   // DeltaNet output projection, K block = the group's head (split-K partial)
  PH_QKV,       // attention q|k|v rows (whole grid)
  PH_ATT,       // split-K flash-decode attention partials (whole grid)
  PH_ATT_OUTP,  // merge of the partials of the group's K block + output projection partial
  PH_GU,        // MLP gate/up rows of the group's K block of the hidden layer
  PH_DOWNP,     // MLP down projection partial over the group's K block
  PH_LM         // final norm + tied LM head rows (whole grid)
};

struct StepArgs {
  DevModel m;         // the engine (by value: read through the constant bank)
  int pos;            // position of this token
  int token;          // input token when tok_src == 0
  int tok_src;        // 1: take the token from amax[amax_in]
  int amax_in, amax_out;
  int st_in, st_out;  // state buffers read / written (distinct)
  float* logits;      // [V] (never NULL: scratch when the caller wants none)
  int32_t* tok_out;   // receives the argmax token (may be NULL)
  float* hidden;      // [n_layers][H] per-layer residual dump (may be NULL)
  uint32_t seq;       // launch sequence number, 1 .. 2^23-1 (tag = seq << 9 | phase)
  int fail_phase;     // debug: phase whose input can never complete (-1 = none)
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


struct PD {                 // one CTA's share of one phase
  const char* p0;           // plane 0 base (row 0 of the phase's row space)
  const char* p1;           // plane 1 base or nullptr
  uint32_t row_bytes;       // bytes of one row of one plane
  int r0, n;                // first row and number of rows of this CTA
  int rpc;                  // rows per chunk
  int keep;                 // 1: L2 evict-last copies (state, KV); 0: evict-first (weights)
  int unit_g, unit_s, S;    // attention split of this CTA (unit_g < 0: none)
};

constexpr int PHASES_PER_LAYER = 5;
constexpr int MAX_PHASES = 128;  // schedule table entries (5 per layer + the LM head)

template <int DK, int HD, int GQ>
struct Cfg {
  static_assert(GQ * HD * 2 + 2 * HD + NCW * GQ * 2 <= UNION_FLOATS, "attention scratch");
  static_assert(4 * DK + 6 <= 2048 && 2048 + 2 * DK <= UNION_FLOATS - 256, "state-phase scratch");
  static constexpr size_t SMEM = size_t(NSLOT) * SLOT + sizeof(SmemTail) +
                                 (UNION_FLOATS + XRAW_MAX) * 4 + MAX_PHASES * sizeof(PD) + 128;
};

// Balanced split of n items into `parts`: [a, b) of part idx.  32-bit
// arithmetic (n * parts < 2^32 for every split the kernel makes).
__device__ __forceinline__ void balanced(int n, int idx, int parts, int& a, int& b) {
  a = int(unsigned(n) * unsigned(idx) / unsigned(parts));
  b = int(unsigned(n) * unsigned(idx + 1) / unsigned(parts));
}

__device__ __forceinline__ int att_splits(const DevModel& M, int pos) {
  int ctx = pos + 1;
  int s = (ctx + ATT_MIN_POS - 1) / ATT_MIN_POS;
  int smax = M.ncta / M.nkv;
  return s < smax ? s : smax;
}

// Group of a CTA (-1 for the CTAs beyond ng * gs) and its rotated index
// inside the group for phase gp (rotation spreads the larger shares).
__device__ __forceinline__ int group_of(const DevModel& M, int cta) {
  return cta < M.ng * M.gs ? cta / M.gs : -1;
}
__device__ __forceinline__ int member_of(const DevModel& M, int cta, int gp) {
  return (cta % M.gs + gp) % M.gs;
}

// One CTA's share of phase gp (layer l, kind).  Evaluated once per launch
// for every phase, by as many threads as there are phases, into the schedule
// table in shared memory that the producer and the consumers walk.
__device__ __noinline__ PD describe(const DevModel& M, const StepArgs& a, int kind, int l,
                                    int gp, int cta) {
  PD d;
  d.p0 = d.p1 = nullptr;
  d.row_bytes = 16;
  d.keep = 0;
  d.unit_g = -1;
  d.unit_s = 0;
  d.S = 0;
  const DevLayer& L = M.layers[l];
  const int grp = group_of(M, cta);
  const int jj = member_of(M, cta, gp);
  int r0 = 0, r1 = 0;
  switch (kind) {
    case PH_DN_IN:
      if (grp >= 0) {
        balanced(M.rin_h, jj, M.gs, r0, r1);
        d.p0 = (const char*)(L.w_in_pk + size_t(grp) * M.rin_h * M.H);
        d.row_bytes = M.H * 2;
      }
      break;
    case PH_DN_ST:
      if (grp >= 0) {
        r0 = 0;
        r1 = M.dv;
        d.p0 = (const char*)(M.dn_state[a.st_in] + (size_t(L.sub) * M.nh + grp) * M.dv * M.dk);
        d.row_bytes = M.dk * 4;
        d.keep = 1;
      }
      break;
    case PH_DN_OUTP:
    case PH_ATT_OUTP: {
      if (grp >= 0) {
        const int kb = kind == PH_DN_OUTP ? M.dv : M.kb_att;
        balanced(M.H, jj, M.gs, r0, r1);
        d.p0 = (const char*)(L.w_out_blk + size_t(grp) * M.H * kb);
        d.row_bytes = kb * 2;
      }
      break;
    }
    case PH_QKV:  // q, k and v rows as one matrix (the engine's packed copy)
      balanced((M.nq + 2 * M.nkv) * M.hd, (cta + gp) % M.ncta, M.ncta, r0, r1);
      d.p0 = (const char*)L.w_qkv;
      d.row_bytes = M.H * 2;
      break;
    case PH_GU:
      if (grp >= 0) {
        balanced(M.kb_mlp, jj, M.gs, r0, r1);
        r0 += grp * M.kb_mlp;
        r1 += grp * M.kb_mlp;
        d.p0 = (const char*)L.w_gate;
        d.p1 = (const char*)L.w_up;
        d.row_bytes = M.H * 2;
      }
      break;
    case PH_DOWNP:
      if (grp >= 0) {
        balanced(M.H, jj, M.gs, r0, r1);
        d.p0 = (const char*)(L.w_down_blk + size_t(grp) * M.H * M.kb_mlp);
        d.row_bytes = M.kb_mlp * 2;
      }
      break;
    case PH_LM:
      balanced(M.V, (cta + gp) % M.ncta, M.ncta, r0, r1);
      d.p0 = (const char*)M.embed;
      d.row_bytes = M.H * 2;
      break;
    case PH_ATT: {
      int S = att_splits(M, a.pos);
      d.S = S;
      d.row_bytes = M.hd * 2;
      d.keep = 1;
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

// Kind and layer of phase gp (PHASES_PER_LAYER per layer, then the LM head).
__device__ __forceinline__ int phase_kind(const DevModel& M, int gp, int& l) {
  l = gp / PHASES_PER_LAYER;
  if (l >= M.n_layers) {
    l = 0;
    return PH_LM;
  }
  static constexpr int dn[PHASES_PER_LAYER] = {PH_DN_IN, PH_DN_ST, PH_DN_OUTP, PH_GU, PH_DOWNP};
  static constexpr int at[PHASES_PER_LAYER] = {PH_QKV, PH_ATT, PH_ATT_OUTP, PH_GU, PH_DOWNP};
  return M.layers[l].is_attn ? at[gp % PHASES_PER_LAYER] : dn[gp % PHASES_PER_LAYER];
}

// Phase sequence of one layer.
__device__ __forceinline__ int layer_phases(const DevLayer& L, int* kinds) {
  if (L.is_attn) {
    kinds[0] = PH_QKV; kinds[1] = PH_ATT; kinds[2] = PH_ATT_OUTP; kinds[3] = PH_GU;
    kinds[4] = PH_DOWNP;
    return 5;
  }
  kinds[0] = PH_DN_IN; kinds[1] = PH_DN_ST; kinds[2] = PH_DN_OUTP; kinds[3] = PH_GU;
  kinds[4] = PH_DOWNP;
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
  return (seq << 9) | uint32_t(phase & 0x1FF);
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
#pragma unroll
  for (int j = 0; j < MAXK; ++j) w[j] = static_cast<unsigned long long>(~tag) << 32;
  uint64_t start = 0;
  for (int it = 0;; ++it) {
#pragma unroll
    for (int j = 0; j < MAXK; ++j) {
      const int i = tid + j * NCT;
      // words already seen complete are not polled again
      if (i >= n) w[j] = static_cast<unsigned long long>(tag) << 32;
      else if (uint32_t(w[j] >> 32) != tag) w[j] = ll_get(src + i);
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

// All NCT consumer threads poll n tagged words (word i at addr(i)) until
// every tag equals `tag`, then store the values to dst[i] (shared memory).
// Each thread keeps its words in registers, so all its loads are in flight
// at once, and re-reads only words still stale.  Uniform result.
template <int MAXK, class AddrFn>
__device__ __forceinline__ bool poll_words(float* dst, int n, AddrFn addr, uint32_t tag,
                                           SmemTail* t, int* err, long long wait_ns, int tid) {
  unsigned long long w[MAXK];
#pragma unroll
  for (int j = 0; j < MAXK; ++j) w[j] = static_cast<unsigned long long>(~tag) << 32;
  uint64_t start = 0;
  for (int it = 0;; ++it) {
#pragma unroll
    for (int j = 0; j < MAXK; ++j) {
      const int i = tid + j * NCT;
      if (i < n && uint32_t(w[j] >> 32) != tag) w[j] = ll_get(addr(i));
    }
    bool stale = false;
#pragma unroll
    for (int j = 0; j < MAXK; ++j) {
      const int i = tid + j * NCT;
      if (i < n) stale |= uint32_t(w[j] >> 32) != tag;
    }
    if (!named_sync_or(1, NCT, stale)) break;
    if (it == 0) start = global_ns();
    else if ((it & 7) == 0 && named_sync_or(1, NCT, give_up(t, err, start, wait_ns)))
      return false;
  }
#pragma unroll
  for (int j = 0; j < MAXK; ++j) {
    const int i = tid + j * NCT;
    if (i < n) dst[i] = __uint_as_float(uint32_t(w[j]));
  }
  return true;
}

// ----------------------------------------------------------------------------
// count-carrying fixed-point sums (the split-K reductions into the residual)
// ----------------------------------------------------------------------------
// Add one contribution y to the word at p.  A contribution outside the
// fixed-point range (or not finite) records MK_ERR_RANGE and adds 0, so the
// count still completes and no reader waits in vain.
__device__ __forceinline__ void cfa_add(unsigned long long* p, float y, int* err) {
  if (!(fabsf(y) < CFA_LIMIT)) {
    record_error(err, MK_ERR_RANGE);
    y = 0.f;
  }
  // y * 2^32 is exact in fp32 (|y| < 2^13), so its float-to-integer
  // rounding is the rounding of y to the 2^-32 grid
  const long long q = __float2ll_rn(y * 4294967296.0f);
  const unsigned long long w =
      (1ull << CFA_SHIFT) + static_cast<unsigned long long>(q + CFA_BIAS);
  asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}

// Consumer threads wait until each of the n words at src counts `want`
// contributions, add the decoded sums to the residual xr[0..n) (shared
// memory), and write xg = xr * gain (the RMSNorm numerator; gv are this
// thread's gains) to xg, returning this thread's sum of xr^2.  Returns false
// in *ok on timeout / abort (per thread; callers agree through
// named_sync_or).
template <int MAXK>
__device__ __forceinline__ float cfa_read_add(float* xr, float* xg, const float* gv,
                                              const unsigned long long* src, int n, int want,
                                              SmemTail* t, int* err, long long wait_ns, int tid,
                                              bool& ok) {
  ok = false;
  if (aborted(t)) return 0.f;
  unsigned long long w[MAXK];
#pragma unroll
  for (int j = 0; j < MAXK; ++j) w[j] = 0;
  uint64_t start = 0;
  for (int it = 0;; ++it) {
#pragma unroll
    for (int j = 0; j < MAXK; ++j) {
      const int i = tid + j * NCT;
      if (i >= n) w[j] = static_cast<unsigned long long>(want) << CFA_SHIFT;
      else if (int(w[j] >> CFA_SHIFT) != want) w[j] = ll_get(src + i);
    }
    bool stale = false;
#pragma unroll
    for (int j = 0; j < MAXK; ++j) stale |= int(w[j] >> CFA_SHIFT) != want;
    if (!stale) break;
    if (it == 0) start = global_ns();
    else if ((it & 7) == 0 && give_up(t, err, start, wait_ns)) return 0.f;
  }
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < MAXK; ++j) {
    const int i = tid + j * NCT;
    if (i < n) {
      const long long q = static_cast<long long>(w[j] & CFA_MASK) - CFA_BIAS * want;
      // the sum is a multiple of 2^-32: one rounding to fp32, exact scaling
      const float v = xr[i] + __ll2float_rn(q) * (1.0f / 4294967296.0f);
      xr[i] = v;
      xg[i] = v * gv[j];
      ss = fmaf(v, v, ss);
    }
  }
  ok = true;
  return ss;
}

// ----------------------------------------------------------------------------
// GEMV helpers (a warp takes up to four rows at a time).  Lane l owns 16-byte
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
enum EpiKind { EPI_STORE, EPI_CFA, EPI_INPROJ, EPI_SWIGLU, EPI_LOGITS };

struct GemvJob {
  PD d;
  int epi;                   // EpiKind
  unsigned long long* dst;   // destination words, indexed by row - dst_off
  int dst_off;
  int* err;                  // EPI_CFA: range errors
  const float4* conv_s;      // EPI_INPROJ: conv history of the CTA's rows (shared memory)
  const uint2* conv_taps;    // EPI_INPROJ: conv taps of the CTA's rows (shared memory)
  float4* conv_out;          // EPI_INPROJ: the layer's conv history in the output state buffer
  int dk, nconv;             // EPI_INPROJ: head rows q|k|v below nconv get the conv
  int chan_q, chan_k, chan_v;  // EPI_INPROJ: conv channels of the head's first q, k, v rows
  int row_b;                 // EPI_INPROJ: packed rows row_b (b) and row_b + 1 (a) become the gates
  float a_log, dt_bias;      // EPI_INPROJ: the head's decay parameters
  float* logits;             // EPI_LOGITS
  float scale;               // multiplies every dot product (the RMSNorm factor)
  uint32_t tag;
};

// Conv channel of packed in-projection row p of one head (p < 2 dk + dv).
__device__ __forceinline__ int conv_channel(const GemvJob& j, int p) {
  return p < j.dk ? j.chan_q + p : p < 2 * j.dk ? j.chan_k + (p - j.dk) : j.chan_v + (p - 2 * j.dk);
}

__device__ __forceinline__ void gemv_epilogue(const GemvJob& j, int row, float y, float y2,
                                              float& best_v, int& best_i) {
  switch (j.epi) {
    case EPI_STORE:
      ll_put(j.dst + (row - j.dst_off), y, j.tag);
      break;
    case EPI_CFA:
      cfa_add(j.dst + (row - j.dst_off), y, j.err);
      break;
    case EPI_INPROJ:
      if (row < j.nconv) {
        // taps (u_{t-3}, u_{t-2}, u_{t-1}, u_t); shift the history by one
        const float4 s = j.conv_s[row - j.d.r0];
        const uint2 wc = j.conv_taps[row - j.d.r0];
        const float c =
            bf_lo(wc.x) * s.x + bf_hi(wc.x) * s.y + bf_lo(wc.y) * s.z + bf_hi(wc.y) * y;
        j.conv_out[conv_channel(j, row)] = make_float4(s.y, s.z, y, 0.f);
        ll_put(j.dst + (row - j.dst_off), siluf_(c), j.tag);
      } else if (row == j.row_b) {
        ll_put(j.dst + (row - j.dst_off), sigmoidf_(y), j.tag);  // beta
      } else if (row == j.row_b + 1) {
        // alpha = exp(-exp(A_log) * softplus(a + dt_bias))
        ll_put(j.dst + (row - j.dst_off), expf(-expf(j.a_log) * softplusf_(y + j.dt_bias)), j.tag);
      } else {
        ll_put(j.dst + (row - j.dst_off), y, j.tag);  // z
      }
      break;
    case EPI_SWIGLU:
      ll_put(j.dst + (row - j.dst_off), siluf_(y) * y2, j.tag);
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
        // as many row dot products as this iteration has rows
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
          if (lane < nb) gemv_epilogue(j, krow, kv * j.scale, kv2 * j.scale, best_v, best_i);
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
  if (lane < nb) gemv_epilogue(j, krow, kv * j.scale, kv2 * j.scale, best_v, best_i);
  if (j.epi == EPI_LOGITS && best_i != 0x7FFFFFFF)
    atomicMax(&t->best, pack_argmax(best_v, best_i));
  return g;
}

// Matrix phases with short rows (the split-K partials, at most 64 16-byte
// vectors per row): LPR lanes share a row, LPR the smallest power of two
// that leaves each lane at most four vectors, so a warp takes 32 / LPR rows
// at a time; the lane's activation slices stay in registers for the phase
// and a row's sum needs log2(LPR) shuffles.
__device__ __forceinline__ uint32_t gemv_short(const GemvJob& j, uint32_t g, unsigned char* ring,
                                               SmemTail* t, int* err, long long wait_ns,
                                               const float* xs) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PD& d = j.d;
  const int nvec = int(d.row_bytes / 16);
  const int LPR = nvec <= 8 ? 2 : nvec <= 16 ? 4 : nvec <= 32 ? 8 : 16;
  const int sl = lane & (LPR - 1), rpp = 32 / LPR, sub = lane / LPR;
  float xr[4][8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int v = sl + LPR * k;
    float4 p = make_float4(0.f, 0.f, 0.f, 0.f), h = p;
    if (v < nvec) {
      p = reinterpret_cast<const float4*>(xs)[v * 2];
      h = reinterpret_cast<const float4*>(xs)[v * 2 + 1];
    }
    xr[k][0] = p.x; xr[k][1] = p.y; xr[k][2] = p.z; xr[k][3] = p.w;
    xr[k][4] = h.x; xr[k][5] = h.y; xr[k][6] = h.z; xr[k][7] = h.w;
  }
  float bv = 0.f;
  int bi = 0;
#pragma unroll 1
  for (int r = d.r0; r < d.r0 + d.n; r += d.rpc, ++g) {
    const int slot = int(g % NSLOT);
    if (bounded_wait(&t->full[slot], (g / NSLOT) & 1, t, err, wait_ns)) {
      const int nr = min(d.rpc, d.r0 + d.n - r);
      const unsigned char* base = ring + size_t(slot) * SLOT;
#pragma unroll 1
      for (int i0 = warp * rpp; i0 < nr; i0 += NCW * rpp) {
        const int i = i0 + sub;
        float a = 0.f, b = 0.f;
        if (i < nr) {
          const uint4* w = reinterpret_cast<const uint4*>(base + size_t(i) * d.row_bytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int v = sl + LPR * k;
            if (v < nvec) fma8x2(w[v], xr[k], a, b);
          }
        }
        float z = a + b;
        for (int o = LPR / 2; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        if (i < nr && sl == 0) gemv_epilogue(j, r + i, z * j.scale, 0.f, bv, bi);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&t->empty[slot]);
  }
  return g;
}

// ----------------------------------------------------------------------------
// RMSNorm: the GEMVs that read a normalised residual take x * gain as their
// activation and scale every dot product by rsqrt(mean(x^2) + eps).
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
// One DeltaNet head's gated delta rule, readout and gated RMSNorm (every CTA
// of the head's group computes the whole head; each writes back its share
// of the new state rows).  Head cache layout in uni (floats), as gathered:
//   [0, DK) q   [DK, 2DK) k   [2DK, 2DK+dv) v   [2DK+dv, 2DK+2dv) z   then
//   beta, alpha (computed by the in-projection epilogue)
//   ov = uni + 2048: readout o (dv)   gv = uni + 2048 + DK: gated output (dv)
// ----------------------------------------------------------------------------
template <int DK>
__device__ __forceinline__ void dn_state_phase(const DevModel& M, const StepArgs& a,
                                               const DevLayer& L, const PD& d, uint32_t& g,
                                               unsigned char* ring, SmemTail* t, float* uni,
                                               uint32_t tag_in, bool dry, int grp, int tid,
                                               int warp, int lane) {
  constexpr int EPL = DK / 32;
  float* hc = uni;
  float* ov = uni + 2048;
  float* gvec = uni + 2048 + DK;
  bool ok = true;
  // the gated norm's gain (element tid), loaded before the wait
  const float wgain = (grp >= 0 && tid < M.dv) ? bf2f(L.out_norm[tid]) : 0.f;
  if (!dry && grp >= 0)
    ok = ll_gather<per_thread(4 * DK + 2)>(hc, M.grp_inp + size_t(grp) * M.rin_h, M.rin_h,
                                           tag_in, t, M.err, a.wait_ns, tid);
  const bool bad = named_sync_or(1, NCT, !ok);
  const bool work = !dry && !bad && grp >= 0;
  // every warp normalises q and k itself (no serial step, no barrier):
  // q, k L2-normalised (eps 1e-6 inside the root), q also scaled by dk^-1/2
  float iq = 0.f, ik = 0.f, kq = 0.f;
  if (work) {
    float sq = 0.f, sk = 0.f, qk = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const float qv = hc[lane * EPL + e], kv = hc[DK + lane * EPL + e];
      sq = fmaf(qv, qv, sq);
      sk = fmaf(kv, kv, sk);
      qk = fmaf(qv, kv, qk);
    }
    sq = warp_sum(sq);
    sk = warp_sum(sk);
    qk = warp_sum(qk);
    iq = 1.0f / sqrtf(sq + 1e-6f) / sqrtf(float(DK));
    ik = 1.0f / sqrtf(sk + 1e-6f);
    kq = qk * iq * ik;
    // w * SiLU(z) of the gated norm, completed after the rows (dv <= NCT)
    if (tid < M.dv) gvec[tid] = wgain * siluf_(hc[2 * DK + M.dv + tid]);
  }
  // this CTA's share of the rows written back (the same split for every
  // launch of the group, unrotated)
  int w0 = 0, w1 = 0;
  if (grp >= 0) balanced(M.dv, int(blockIdx.x) % M.gs, M.gs, w0, w1);
  float* st = M.dn_state[a.st_out] + (size_t(L.sub) * M.nh + (grp < 0 ? 0 : grp)) * M.dv * DK;
  const float beta = hc[4 * DK], alpha = hc[4 * DK + 1];  // gates from the in-projection
  // The head's dv rows are one ring chunk.  Eight lanes share a row (a warp
  // takes four rows at a time); sub-lane sl owns the float4 columns
  // sl, sl + 8, ... so a row's eight lanes read consecutive 16-byte words
  // (no bank conflicts), and k and q for those columns stay in registers.
  constexpr int LPR = 8, V4 = DK / (4 * LPR);
  const int sl = lane & (LPR - 1), ro = lane / LPR;
  float4 kk[V4], qq[V4];
#pragma unroll
  for (int k = 0; k < V4; ++k) {
    const float4 kr = reinterpret_cast<const float4*>(hc + DK)[sl + LPR * k];
    const float4 qr = reinterpret_cast<const float4*>(hc)[sl + LPR * k];
    kk[k] = make_float4(kr.x * ik, kr.y * ik, kr.z * ik, kr.w * ik);
    qq[k] = make_float4(qr.x * iq, qr.y * iq, qr.z * iq, qr.w * iq);
  }
  float oss = 0.f;  // this lane's rows' o^2 (lanes with sl == 0)
  if (d.n > 0) {
    const int slot = int(g % NSLOT);
    const bool okw = bounded_wait(&t->full[slot], (g / NSLOT) & 1, t, M.err, a.wait_ns);
    if (okw && work) {
      const float* base = reinterpret_cast<const float*>(ring + size_t(slot) * SLOT);
      for (int r0 = warp * 4; r0 < d.n; r0 += NCW * 4) {
        const int row = r0 + ro;
        const bool has = row < d.n;
        float4 sv[V4];
        float s_k = 0.f, s_q = 0.f;
#pragma unroll
        for (int k = 0; k < V4; ++k) {
          sv[k] = has ? reinterpret_cast<const float4*>(base + size_t(row) * DK)[sl + LPR * k]
                      : make_float4(0.f, 0.f, 0.f, 0.f);
          s_k = fmaf(sv[k].x, kk[k].x, s_k);
          s_k = fmaf(sv[k].y, kk[k].y, s_k);
          s_k = fmaf(sv[k].z, kk[k].z, s_k);
          s_k = fmaf(sv[k].w, kk[k].w, s_k);
          s_q = fmaf(sv[k].x, qq[k].x, s_q);
          s_q = fmaf(sv[k].y, qq[k].y, s_q);
          s_q = fmaf(sv[k].z, qq[k].z, s_q);
          s_q = fmaf(sv[k].w, qq[k].w, s_q);
        }
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) {
          s_k += __shfl_xor_sync(0xffffffffu, s_k, o);
          s_q += __shfl_xor_sync(0xffffffffu, s_q, o);
        }
        if (has) {
          const float u = beta * (hc[2 * DK + row] - alpha * s_k);  // S' = alpha S + u k^T
          if (row >= w0 && row < w1) {
            float4* dst = reinterpret_cast<float4*>(st + size_t(row) * DK);
#pragma unroll
            for (int k = 0; k < V4; ++k)
              dst[sl + LPR * k] = make_float4(fmaf(alpha, sv[k].x, u * kk[k].x),
                                              fmaf(alpha, sv[k].y, u * kk[k].y),
                                              fmaf(alpha, sv[k].z, u * kk[k].z),
                                              fmaf(alpha, sv[k].w, u * kk[k].w));
          }
          if (sl == 0) {
            const float o = fmaf(alpha, s_q, u * kq);  // o_i = S'_i . q
            ov[row] = o;
            oss = fmaf(o, o, oss);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&t->empty[slot]);
    ++g;
  }
  oss = warp_sum(oss);
  if (lane == 0) t->red[warp] = oss;
  const bool skip = named_sync_or(1, NCT, !work || aborted(t));
  if (skip) return;
  // gated RMSNorm of the head's readout: g = o * rsqrt(mean(o^2) + eps) * w * SiLU(z)
  float ss = 0.f;
#pragma unroll
  for (int w = 0; w < NCW; ++w) ss += t->red[w];
  const float inv = 1.0f / sqrtf(ss / float(M.dv) + M.eps);
  if (tid < M.dv) gvec[tid] *= ov[tid] * inv;
  named_sync(1, NCT);
}

// EPL consecutive bf16 values (16, 8 or 4 bytes, aligned) as floats.
template <int EPL>
__device__ __forceinline__ void load_bf16_vec(const uint16_t* p, float (&f)[EPL]) {
  if constexpr (EPL == 8) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    f[0] = bf_lo(u.x); f[1] = bf_hi(u.x); f[2] = bf_lo(u.y); f[3] = bf_hi(u.y);
    f[4] = bf_lo(u.z); f[5] = bf_hi(u.z); f[6] = bf_lo(u.w); f[7] = bf_hi(u.w);
  } else if constexpr (EPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    f[0] = bf_lo(u.x); f[1] = bf_hi(u.x); f[2] = bf_lo(u.y); f[3] = bf_hi(u.y);
  } else {
    static_assert(EPL == 2, "head_dim 64, 128 or 256");
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    f[0] = bf_lo(u); f[1] = bf_hi(u);
  }
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
// split-K flash-decode attention for one KV group and position range: the
// CTA's partial (per q head of the group: accumulator, running max m and
// denominator l) is published as tagged words; the merge happens in the
// output-projection phase (att_merge_block).
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
  // The chunk loop keeps the last ring slot: once its cached positions are
  // consumed it is the scratch where the warps' partials are combined.
  int keep_slot = -1;
  {
    int local_ = 0;
    for (int r_ = d.r0; r_ < d.r0 + d.n; r_ += d.rpc, ++g, local_ += d.rpc) {
      const int slot_ = int(g % NSLOT);
      const bool ok_ = bounded_wait(&t->full[slot_], (g / NSLOT) & 1, t, M.err, a.wait_ns);
      if (ok_) {
        const int nr_ = min(d.rpc, d.r0 + d.n - r_);
        const unsigned char* base_ = ring + size_t(slot_) * SLOT;
        for (int i_ = (warp - (local_ % NCW) + NCW) % NCW; i_ < nr_; i_ += NCW) {
          float kf[EPL], vf[EPL];
          load_bf16_vec<EPL>(reinterpret_cast<const uint16_t*>(base_ + size_t(i_) * d.row_bytes) +
                                 lane * EPL,
                             kf);
          load_bf16_vec<EPL>(
              reinterpret_cast<const uint16_t*>(base_ + size_t(d.rpc + i_) * d.row_bytes) +
                  lane * EPL,
              vf);
          att_consume<G, EPL>(am, al, acc, qr, kf, vf, scale);
        }
      }
      __syncwarp();
      if (r_ + d.rpc < d.r0 + d.n) {
        if (lane == 0) mbar_arrive(&t->empty[slot_]);
      } else {
        keep_slot = slot_;
      }
    }
  }
  const bool go = !named_sync_or(1, NCT, aborted(t) || !work);
  if (go) {
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
    float fw[G];
#pragma unroll
    for (int j = 0; j < G; ++j) {
      float mx = -INFINITY;
      for (int w = 0; w < NCW; ++w) mx = fmaxf(mx, att_ml[(w * G + j) * 2]);
      fw[j] = al[j] > 0.f ? expf(am[j] - mx) : 0.f;
    }
    // publish this split's partial as tagged words: per head [acc(HD) | m | l]
    unsigned long long* pbase =
        M.part_ll + (size_t(gidx) * kMaxCtas + d.unit_s) * G * (HD + 2);
    if (keep_slot >= 0) {
      // every warp's rescaled accumulator to the kept slot ([warp][head][HD],
      // element lane*EPL + e at e*32 + lane: conflict-free), then one sum per
      // element in warp order (deterministic)
      float* scr = reinterpret_cast<float*>(ring + size_t(keep_slot) * SLOT);
#pragma unroll
      for (int j = 0; j < G; ++j)
#pragma unroll
        for (int e = 0; e < EPL; ++e) scr[(warp * G + j) * HD + e * 32 + lane] = fw[j] * acc[j][e];
      named_sync(1, NCT);
      for (int off = tid; off < G * HD; off += NCT) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < NCW; ++w) sum += scr[w * G * HD + off];
        const int j = off / HD, rem = off % HD;
        ll_put(pbase + j * (HD + 2) + (rem % 32) * EPL + rem / 32, sum, tag_out);
      }
    } else if (warp == 0) {
      // no cached positions: warp 0 alone holds the new position
#pragma unroll
      for (int j = 0; j < G; ++j)
#pragma unroll
        for (int e = 0; e < EPL; ++e)
          ll_put(pbase + j * (HD + 2) + lane * EPL + e, fw[j] * acc[j][e], tag_out);
    }
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
  }
  // release the kept slot once every warp is done with it
  if (keep_slot >= 0) {
    named_sync(1, NCT);
    if (lane == 0) mbar_arrive(&t->empty[keep_slot]);
  }
}

// ----------------------------------------------------------------------------
// Merge the attention partials of all S splits for elements [e0, e0 + kb) of
// the concatenated head outputs (nq * hd) into ov (shared memory), in a fixed
// split order: o_e = sum_s exp(m_s - m) acc_s[e] / sum_s exp(m_s - m) l_s,
// per q head.  Scratch in uni: staged values [0, MERGE_STAGE), then (m, l)
// and weights of every split for each head the block touches.
// ----------------------------------------------------------------------------
template <int HD, int GQ>
__device__ __forceinline__ bool att_merge_block(const DevModel& M, int S, int e0, int kb,
                                                float* uni, float* ov, uint32_t tag,
                                                SmemTail* t, int* err, long long wait_ns,
                                                int tid) {
  const int h_lo = e0 / HD, nhb = (e0 + kb - 1) / HD - h_lo + 1;
  float* stage = uni;
  float* mls = uni + MERGE_STAGE;        // [S][nhb][2]
  float* wgt = mls + 2 * S * nhb;        // [S][nhb]
  // address of element c (< HD: accumulator, HD: m, HD + 1: l) of q head hq, split si
  auto part = [&](int si, int hq, int c) {
    return M.part_ll + ((size_t(hq / GQ) * kMaxCtas + si) * GQ + hq % GQ) * (HD + 2) + c;
  };
  // (m, l) of every split for the block's heads
  if (!poll_words<per_thread(MERGE_ML_MAX)>(
          mls, S * nhb * 2,
          [&](int w) { return part(w / (nhb * 2), h_lo + (w >> 1) % nhb, HD + (w & 1)); }, tag, t,
          err, wait_ns, tid))
    return false;
  if (tid < nhb) {
    float mx = -INFINITY;
    for (int si = 0; si < S; ++si) mx = fmaxf(mx, mls[(si * nhb + tid) * 2]);
    float den = 0.f;
    for (int si = 0; si < S; ++si) {
      const float f = expf(mls[(si * nhb + tid) * 2] - mx);
      wgt[si * nhb + tid] = f;
      den = fmaf(f, mls[(si * nhb + tid) * 2 + 1], den);
    }
    const float inv = 1.0f / den;
    for (int si = 0; si < S; ++si) wgt[si * nhb + tid] *= inv;
  }
  for (int e = tid; e < kb; e += NCT) ov[e] = 0.f;
  named_sync(1, NCT);
  // accumulator values, a batch of splits at a time
  const int sb_max = MERGE_STAGE / kb;
  for (int s0 = 0; s0 < S; s0 += sb_max) {
    const int sb = min(sb_max, S - s0);
    if (!poll_words<per_thread(MERGE_STAGE)>(
            stage, sb * kb,
            [&](int w) {
              const int e = e0 + w % kb;
              return part(s0 + w / kb, e / HD, e % HD);
            },
            tag, t, err, wait_ns, tid))
      return false;
    for (int e = tid; e < kb; e += NCT) {
      const int hb = (e0 + e) / HD - h_lo;
      float o = ov[e];
      for (int q = 0; q < sb; ++q) o = fmaf(wgt[(s0 + q) * nhb + hb], stage[q * kb + e], o);
      ov[e] = o;
    }
    named_sync(1, NCT);
  }
  return true;
}

// ----------------------------------------------------------------------------
// Cursor over one CTA's chunk schedule for one launch: every phase of every
// layer, then the LM head, each split into chunks of at most `rpc` rows.
// ----------------------------------------------------------------------------
constexpr size_t PF_AHEAD = size_t(128) << 10;  // L2 prefetch distance per CTA (bytes)

struct ChunkCursor {
  const PD* tab;
  int np;     // phases in the launch
  int gp;     // current phase
  int r;      // first row of the current chunk
  bool done;
  __device__ __forceinline__ const PD& d() const { return tab[gp]; }
  __device__ __forceinline__ int nrows() const { return min(d().rpc, d().r0 + d().n - r); }
  __device__ __forceinline__ uint32_t bytes() const { return uint32_t(nrows()) * d().row_bytes; }
  __device__ __forceinline__ const char* src0() const { return d().p0 + size_t(r) * d().row_bytes; }
  __device__ __forceinline__ const char* src1() const { return d().p1 + size_t(r) * d().row_bytes; }
};

// Move to the first chunk at or after phase gp; skips empty phases.
__device__ __forceinline__ void cursor_settle(ChunkCursor& c) {
  while (c.gp < c.np && c.tab[c.gp].n == 0) ++c.gp;
  c.done = c.gp >= c.np;
  if (!c.done) c.r = c.tab[c.gp].r0;
}

__device__ __forceinline__ void cursor_init(ChunkCursor& c, const PD* tab, int np) {
  c.tab = tab;
  c.np = np;
  c.gp = 0;
  cursor_settle(c);
}

__device__ __forceinline__ void cursor_next(ChunkCursor& c) {
  c.r += c.d().rpc;
  if (c.r < c.d().r0 + c.d().n) return;
  ++c.gp;
  cursor_settle(c);
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
  float* xraw = uni + UNION_FLOATS;  // the residual stream (identical in every CTA)
  PD* tab = reinterpret_cast<PD*>(xraw + XRAW_MAX);  // this CTA's schedule, one entry per phase

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
  // The schedule: this CTA's share of every phase, one phase per thread.
  const int n_phases = M.n_layers * PHASES_PER_LAYER + 1;
  for (int i = tid; i < n_phases; i += NTHR) {
    int l;
    const int kind = phase_kind(M, i, l);
    tab[i] = describe(M, a, kind, l, i, cta);
  }
  // RoPE table for this position (angles in double: pos * theta^(-2i/hd)).
  for (int i = tid; i < HD / 2; i += NTHR) {
    double inv_freq = pow(double(M.theta), -2.0 * double(i) / double(HD));
    double s, c;
    sincos(double(a.pos) * inv_freq, &s, &c);
    t->rope_cos[i] = float(c);
    t->rope_sin[i] = float(s);
  }
  // Clear this CTA's share of the other launch parity's sum words: the next
  // launch adds into them (this launch adds into its own parity's words,
  // cleared by the launch before it or by mk_reset).
  const size_t xacc_words = size_t(M.n_layers) * 2 * M.H;
  {
    unsigned long long* other = M.xacc + size_t((a.seq & 1u) ^ 1u) * xacc_words;
    const size_t z0 = xacc_words * cta / M.ncta, z1 = xacc_words * (cta + 1) / M.ncta;
    for (size_t i = z0 + tid; i < z1; i += NTHR) other[i] = 0ull;
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
    cursor_init(ld, tab, n_phases);
    cursor_init(pf, tab, n_phases);
    size_t ld_bytes = 0, pf_bytes = 0;
    uint32_t g = 0;
    while (!ld.done && !aborted(t)) {
      // keep the prefetch cursor PF_AHEAD bytes ahead of the loads
      while (!pf.done && pf_bytes < ld_bytes + PF_AHEAD) {
        const uint32_t b = pf.bytes();
        bulk_prefetch_l2(pf.src0(), b);
        if (pf.d().p1) bulk_prefetch_l2(pf.src1(), b);
        pf_bytes += size_t(b) * (pf.d().p1 ? 2 : 1);
        cursor_next(pf);
      }
      const int slot = int(g % NSLOT);
      if (g >= NSLOT && !bounded_wait(&t->empty[slot], ((g / NSLOT) - 1) & 1, t, M.err, a.wait_ns))
        break;
      const uint32_t bytes = ld.bytes();
      unsigned char* dst = ring + size_t(slot) * SLOT;
      const PD& ldd = ld.d();
      const uint64_t pol = ldd.keep ? pol_s : pol_w;
      mbar_arrive_expect_tx(&t->full[slot], bytes * (ldd.p1 ? 2u : 1u));
      bulk_g2s(dst, ld.src0(), bytes, &t->full[slot], pol);
      if (ldd.p1)
        bulk_g2s(dst + size_t(ldd.rpc) * ldd.row_bytes, ld.src1(), bytes, &t->full[slot], pol);
      ld_bytes += size_t(bytes) * (ldd.p1 ? 2 : 1);
      ++g;
      cursor_next(ld);
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
  const int grp = group_of(M, cta);
  unsigned long long* xacc = M.xacc + size_t(a.seq & 1u) * xacc_words;  // [n_layers][2][H]
  uint32_t g = 0;  // chunk counter (same order as the producer)
  int gp = 0;
  int kinds[8];
  uint32_t tag_qkv = 0, tag_att = 0;  // producers of the attention exchanges
  uint32_t tag_inp = 0, tag_h = 0;    // producers of the group exchanges
  float* ovec = uni + UNION_FLOATS - 256;  // merged attention block (<= 256 floats)

  // the residual stream starts as the token's embedding row (every CTA)
  {
    const uint16_t* emb_row = M.embed + size_t(tok) * M.H;
    for (int i = tid; i < M.H; i += NCT) xraw[i] = bf2f(emb_row[i]);
  }

  for (int l = 0; l <= M.n_layers; ++l) {
    const bool lm = (l == M.n_layers);
    const DevLayer& L = M.layers[lm ? 0 : l];
    int np;
    if (!lm) np = layer_phases(L, kinds);
    else { kinds[0] = PH_LM; np = 1; }

    for (int p = 0; p < np; ++p, ++gp) {
      const int kind = kinds[p];
      const PD d = tab[gp];
      const uint32_t tag_me = make_tag(a.seq, gp);
      // debug hook: the inputs of phase `fail_phase` can never complete
      const bool fail_here = gp == a.fail_phase;
      const uint32_t dbg = fail_here ? 0x80000000u : 0u;
      const int want = M.ng + (fail_here ? 1 : 0);
      // uniform across the consumer warps (also orders the previous phase)
      const bool dry = named_sync_or(1, NCT, aborted(t));
      GemvJob j{};  // matrix phases fill it in; one dispatch after the switch
      j.d = d;
      j.tag = tag_me;
      j.err = M.err;
      j.scale = 1.f;
      bool gemv = false;
      const float* xs = uni;
      switch (kind) {
        case PH_DN_IN:
        case PH_QKV:
        case PH_GU:
        case PH_LM: {
          // input: the residual stream completed by the previous split-K sum
          // (none before layer 0), then its RMSNorm
          bool ok = true;
          // union layout in this phase: x [0, 2048) | conv history [2048, 3072)
          // (<= CONV_ROWS_MAX float4) | conv taps [3072, 3584) (<= CONV_ROWS_MAX uint2)
          float4* conv_s = reinterpret_cast<float4*>(uni + 2048);
          uint2* conv_taps = reinterpret_cast<uint2*>(uni + 2048 + 4 * CONV_ROWS_MAX);
          const uint16_t* gain = kind == PH_GU ? L.mlp_norm
                                 : kind == PH_LM ? M.final_norm : L.attn_norm;
          float gv[GK];
          load_gains(gv, gain, M.H, tid);
          float ss = 0.f;
          const int src_layer = kind == PH_GU ? l : l - 1;
          const int src_half = kind == PH_GU ? 0 : 1;
          if (!dry) {
            if (kind == PH_DN_IN && grp >= 0) {
              // stage the conv history and taps of this CTA's q|k|v rows first
              // (independent of the input: their latency overlaps the wait)
              const int nconv = max(0, min(d.r0 + d.n, 2 * M.dk + M.dv) - d.r0);
              const float4* conv_in =
                  reinterpret_cast<const float4*>(M.conv_state[a.st_in]) + size_t(L.sub) * M.ch;
              GemvJob cj{};
              cj.dk = M.dk;
              cj.chan_q = grp * M.dk;
              cj.chan_k = M.nh * M.dk + grp * M.dk;
              cj.chan_v = 2 * M.nh * M.dk + grp * M.dv;
              for (int i = tid; i < nconv; i += NCT) {
                const int ch = conv_channel(cj, d.r0 + i);
                conv_s[i] = conv_in[ch];
                conv_taps[i] = *reinterpret_cast<const uint2*>(L.conv_w + size_t(ch) * 4);
              }
            }
            // the residual stream (completed by the split-K sum) and x * gain,
            // the RMSNorm numerator; the GEMV scales its results by the norm
            if (src_layer >= 0) {
              ss = cfa_read_add<GK>(xraw, uni, gv,
                                    xacc + (size_t(src_layer) * 2 + src_half) * M.H, M.H, want,
                                    t, M.err, a.wait_ns, tid, ok);
            } else {
#pragma unroll
              for (int k = 0; k < GK; ++k) {
                const int i = tid + k * NCT;
                if (i < M.H) {
                  const float v = xraw[i];
                  uni[i] = v * gv[k];
                  ss = fmaf(v, v, ss);
                }
              }
            }
          }
          ss = warp_sum(ss);
          if (lane == 0) t->red[warp] = ss;
          const bool bad = named_sync_or(1, NCT, !ok);
          if (!dry && !bad) {
            if (src_half == 1 && src_layer >= 0 && cta == 0 && a.hidden)
              for (int i = tid; i < M.H; i += NCT) a.hidden[size_t(src_layer) * M.H + i] = xraw[i];
            float tot = 0.f;
#pragma unroll
            for (int w = 0; w < NCW; ++w) tot += t->red[w];
            j.scale = 1.0f / sqrtf(tot / float(M.H) + M.eps);
          }
          gemv = true;
          if (kind == PH_DN_IN) {
            j.epi = EPI_INPROJ;
            j.dst = M.grp_inp + size_t(grp < 0 ? 0 : grp) * M.rin_h;
            j.conv_s = conv_s;
            j.conv_taps = conv_taps;
            j.conv_out = reinterpret_cast<float4*>(M.conv_state[a.st_out]) + size_t(L.sub) * M.ch;
            j.dk = M.dk;
            j.nconv = 2 * M.dk + M.dv;
            j.chan_q = grp * M.dk;
            j.chan_k = M.nh * M.dk + grp * M.dk;
            j.chan_v = 2 * M.nh * M.dk + grp * M.dv;
            j.row_b = 2 * M.dk + 2 * M.dv;
            j.a_log = grp >= 0 ? L.A_log[grp] : 0.f;
            j.dt_bias = grp >= 0 ? L.dt_bias[grp] : 0.f;
            tag_inp = tag_me;
          } else if (kind == PH_QKV) {
            j.epi = EPI_STORE;
            j.dst = M.qkv_ll;  // [q | k | v], the rows' order
            tag_qkv = tag_me;
          } else if (kind == PH_GU) {
            j.epi = EPI_SWIGLU;
            j.dst = M.grp_h + size_t(grp < 0 ? 0 : grp) * M.kb_mlp;
            j.dst_off = (grp < 0 ? 0 : grp) * M.kb_mlp;
            tag_h = tag_me;
          } else {
            j.epi = EPI_LOGITS;
            j.logits = a.logits;
          }
          break;
        }
        case PH_DN_ST:
          dn_state_phase<DK>(M, a, L, d, g, ring, t, uni, tag_inp | dbg, dry, grp, tid, warp,
                             lane);
          break;
        case PH_DN_OUTP:
          // the head's gated output (left in uni + 2048 + DK by the state
          // phase) times the head's K block of the output projection
          gemv = true;
          xs = uni + 2048 + DK;
          j.epi = EPI_CFA;
          j.dst = xacc + (size_t(l) * 2 + 0) * M.H;
          break;
        case PH_ATT:
          attention_phase<HD, GQ>(M, a, L, d, g, ring, t, uni, tag_qkv, dbg, tag_me, dry, tid,
                                  warp, lane);
          tag_att = tag_me;
          break;
        case PH_ATT_OUTP: {
          bool ok = true;
          if (!dry && grp >= 0)
            ok = att_merge_block<HD, GQ>(M, att_splits(M, a.pos), grp * M.kb_att, M.kb_att, uni,
                                         ovec, tag_att | dbg, t, M.err, a.wait_ns, tid);
          named_sync_or(1, NCT, !ok);
          gemv = true;
          xs = ovec;
          j.epi = EPI_CFA;
          j.dst = xacc + (size_t(l) * 2 + 0) * M.H;
          break;
        }
        case PH_DOWNP: {
          // the group's K block of SiLU(gate)*up, then the down-projection partial
          bool ok = true;
          if (!dry && grp >= 0)
            ok = ll_gather<per_thread(UNION_FLOATS)>(uni, M.grp_h + size_t(grp) * M.kb_mlp,
                                                     M.kb_mlp, tag_h | dbg, t, M.err, a.wait_ns,
                                                     tid);
          named_sync_or(1, NCT, !ok);
          gemv = true;
          j.epi = EPI_CFA;
          j.dst = xacc + (size_t(l) * 2 + 1) * M.H;
          break;
        }
        default:
          break;
      }
      if (gemv)
        g = (j.epi == EPI_CFA && d.row_bytes <= 1024)
                ? gemv_short(j, g, ring, t, M.err, a.wait_ns, xs)
                : gemv_core(j, g, ring, t, M.err, a.wait_ns, xs);
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
