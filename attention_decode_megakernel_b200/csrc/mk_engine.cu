// mk_engine.cu -- host side of the C ABI declared in include/mk.h: config
// validation, workspace carve-up, cooperative launches of the decode kernel,
// state buffer rotation, verify records and their replay, state I/O and error
// reporting.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <new>
#include <utility>

#include "mk.h"
#include "mk_chunk.cuh"
#include "mk_decode.cuh"
#include "mk_delta.cuh"
#include "mk_model.cuh"
#include "mk_prefill.cuh"
#include "mk_skinny.cuh"
#include "mk_lowbit.cuh"
#include "mk_verify.cuh"

namespace {

using mk::DevModel;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Layout {
  size_t model;
  size_t dn_state[mk::kStateBufs], conv_state[mk::kStateBufs];
  size_t kc, vc;
  size_t xacc, grp_inp, grp_h, qkv, part, hidden, logits, tickets, err, amax;
  // weight copies laid out for the decode kernel's groups
  size_t wqkv;      // q|k|v rows of every attention layer
  size_t w_in_pk;   // DeltaNet in-projection rows per head
  size_t w_out_blk; // output projections by K block
  size_t w_down_blk;  // MLP down projections by K block
  // multi-token prompt path: T_MAX positions per chunk
  int tmax, pw, aw;
  size_t pf_tok, pf_x, pf_xn, pf_p, pf_c, pf_o, pf_a16, pf_qk, pf_bak, pf_att, pf_part;
  size_t pf_chunk;  // chunkwise delta rule operands: [nh][chunks][block]
  // verify records, two sets: keys, values [n_dn][kMaxVerify][nh][dk],
  // {alpha, beta} [n_dn][kMaxVerify][nh], conv inputs [n_dn][kMaxVerify][ch]
  size_t vlog_k[2], vlog_v[2], vlog_ab[2], vlog_u[2];
  size_t total;
};

constexpr int kPrefillChunk = 1024;  // most positions one prompt chunk processes
constexpr int kPrefillMinBatch = 8;  // shorter prompts run as decode steps
constexpr int kSplitMaxTiles = 100;      // prompt GEMMs with fewer output tiles split K
constexpr int kSplitPartialTiles = 148 + kSplitMaxTiles;

int count_attn(const mk_config& c) {
  int n = 0;
  for (int l = 0; l < c.n_layers; ++l) n += c.layer_is_attn[l] ? 1 : 0;
  return n;
}

bool basic_valid(const mk_config* c) {
  if (!c) return false;
  if (c->n_layers < 1 || c->n_layers > MK_MAX_LAYERS) return false;
  if (c->hidden <= 0 || c->vocab <= 0 || c->mlp <= 0) return false;
  if (c->dn_heads <= 0 || c->dn_dk <= 0 || c->dn_dv <= 0 || c->conv_k <= 0) return false;
  if (c->q_heads <= 0 || c->kv_heads <= 0 || c->head_dim <= 0) return false;
  if (c->max_ctx <= 0 || c->max_verify <= 0 || c->max_verify > mk::kMaxVerify) return false;
  if (c->q_heads % c->kv_heads) return false;
  return true;
}

Layout make_layout(const mk_config& c) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const int n_attn = count_attn(c), n_dn = c.n_layers - n_attn;
  const size_t ch = size_t(2) * c.dn_heads * c.dn_dk + size_t(c.dn_heads) * c.dn_dv;
  const size_t rin = ch + size_t(c.dn_heads) * c.dn_dv + 2 * size_t(c.dn_heads);
  const size_t G = size_t(c.q_heads / c.kv_heads);
  L.model = take(sizeof(DevModel));
  for (int b = 0; b < mk::kStateBufs; ++b) {
    L.dn_state[b] = take(size_t(n_dn) * c.dn_heads * c.dn_dv * c.dn_dk * 4);
    L.conv_state[b] = take(size_t(n_dn) * ch * 4 * 4);
  }
  const size_t kv = size_t(n_attn) * c.kv_heads * c.max_ctx * c.head_dim * 2;
  L.kc = take(kv);
  L.vc = take(kv);
  L.wqkv = take(size_t(n_attn) * (c.q_heads + 2 * c.kv_heads) * c.head_dim * c.hidden * 2);
  const size_t rin_h = 2 * size_t(c.dn_dk) + 2 * size_t(c.dn_dv) + 2;
  L.w_in_pk = take(size_t(n_dn) * c.dn_heads * rin_h * c.hidden * 2);
  {
    size_t outw = 0;  // K of every layer's output projection
    for (int l = 0; l < c.n_layers; ++l)
      outw += c.layer_is_attn[l] ? size_t(c.q_heads) * c.head_dim : size_t(c.dn_heads) * c.dn_dv;
    L.w_out_blk = take(outw * c.hidden * 2);
  }
  L.w_down_blk = take(size_t(c.n_layers) * c.hidden * c.mlp * 2);
  L.xacc = take(size_t(2) * c.n_layers * 2 * c.hidden * 8);
  L.grp_inp = take(size_t(c.dn_heads) * rin_h * 8);
  L.grp_h = take(size_t(c.mlp + c.dn_heads) * 8);
  L.qkv = take(size_t(c.q_heads + 2 * c.kv_heads) * c.head_dim * 8);
  L.part = take(size_t(c.kv_heads) * mk::kMaxCtas * G * (c.head_dim + 2) * 8);
  L.hidden = take(size_t(c.n_layers) * c.hidden * 4);
  L.logits = take(size_t(c.vocab) * 4);
  L.tickets = take(4);
  L.err = take(4);
  L.amax = take(2 * 8);
  {
    const int T = c.max_ctx < kPrefillChunk ? c.max_ctx : kPrefillChunk;
    const int nqkv = (c.q_heads + 2 * c.kv_heads) * c.head_dim;
    int pw = int(rin);
    if (2 * c.mlp > pw) pw = 2 * c.mlp;
    if (nqkv > pw) pw = nqkv;
    int aw = c.dn_heads * c.dn_dv;
    if (c.mlp > aw) aw = c.mlp;
    if (c.q_heads * c.head_dim > aw) aw = c.q_heads * c.head_dim;
    L.tmax = T;
    L.pw = pw;
    L.aw = aw;
    L.pf_tok = take(size_t(T) * 4);
    L.pf_x = take(size_t(T) * c.hidden * 4);
    L.pf_xn = take(size_t(2) * T * c.hidden * 2);  // [hi|lo][T][H] bf16
    L.pf_p = take(size_t(T) * pw * 4);
    L.pf_c = take(size_t(T) * ch * 4);  // conv output of the q|k|v channels
    L.pf_o = take(size_t(T) * c.dn_heads * c.dn_dv * 4);
    L.pf_a16 = take(size_t(2) * T * aw * 2);  // [hi|lo][T][aw] bf16
    L.pf_qk = take(size_t(c.dn_heads) * T * 2 * c.dn_dk * 4);
    L.pf_bak = take(size_t(c.dn_heads) * T * 16);
    // key-split attention partials of a short chunk: [t][q head][range][hd + 2]
    const size_t rlen = mk::pf::ATT_SPLIT_LEN < mk::vf::ATT_L ? mk::pf::ATT_SPLIT_LEN : mk::vf::ATT_L;
    const size_t nsplit = (size_t(c.max_ctx) + rlen - 1) / rlen;
    L.pf_att = take(size_t(mk::kMaxVerify) * c.q_heads * nsplit * (c.head_dim + 2) * 4);
    // split-K partial sums of a prompt GEMM with few output tiles (< 100):
    // k_split x T x n_out <= (148 + tiles) x 128 x 128 floats
    L.pf_part = take(size_t(kSplitPartialTiles) * mk::pf::BM * mk::pf::BN * 4);
    const size_t blk = c.dn_dk == 64 ? mk::ck::Blk<64>::FLOATS : mk::ck::Blk<128>::FLOATS;
    L.pf_chunk = take(size_t(c.dn_heads) * ((T + mk::ck::C - 1) / mk::ck::C) * blk * 4);
  }
  {
    const size_t n_dn = size_t(c.n_layers - count_attn(c)), V = mk::kMaxVerify;
    for (int sel = 0; sel < 2; ++sel) {
      L.vlog_k[sel] = take(n_dn * V * c.dn_heads * c.dn_dk * 4);
      L.vlog_v[sel] = take(n_dn * V * c.dn_heads * c.dn_dv * 4);
      L.vlog_ab[sel] = take(n_dn * V * c.dn_heads * 8);
      L.vlog_u[sel] = take(n_dn * V * ch * 4);
    }
  }
  L.total = off;
  return L;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

// 2D bf16 matrix [rows][cols] (row pitch in elements) as TMA tiles of
// box_rows x 64 columns with the 128-byte swizzle the MMA descriptors expect.
bool make_map(CUtensorMap* m, const void* base, int rows, int cols, int pitch, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || (reinterpret_cast<uintptr_t>(base) & 15u) || cols % 64 || (pitch * 2) % 16)
    return false;
  const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(pitch) * 2};
  const cuuint32_t box[2] = {64u, cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Variant {
  int dk, hd, g;
  const void* fn;
  size_t smem;
};

template <int DK, int HD, int GQ>
Variant variant() {
  return Variant{DK, HD, GQ, reinterpret_cast<const void*>(&mk::decode_kernel<DK, HD, GQ>),
                 mk::Cfg<DK, HD, GQ>::SMEM};
}

const Variant* find_variant(int dk, int hd, int g) {
  static const Variant table[] = {
      variant<64, 64, 4>(),
      variant<128, 256, 4>(),
      variant<128, 128, 4>(),
  };
  for (const Variant& v : table)
    if (v.dk == dk && v.hd == hd && v.g == g) return &v;
  return nullptr;
}

}  // namespace

struct mk_engine {
  mk_config cfg;
  int device;
  cudaStream_t stream;
  char* ws;
  Layout lay;
  DevModel hm;  // host copy of the device model
  DevModel* dm;
  const Variant* var;
  int ncta;
  int pos;
  int cur_buf;
  uint32_t seq;  // launch sequence number for activation tags
  int amax_toggle;
  bool amax_valid;  // the last launch was a decode step at the current position
  int pending_verify;
  int verify_bufs[mk::kMaxVerify];
  // verify by records (the chunk path): the pending verify wrote record set
  // vlog_sel; after mk_accept the first replay_n records of set replay_sel
  // are applied to the state by the next call that reads it
  bool verify_logged;
  int vlog_sel, replay_n, replay_sel;
  int64_t launches;
  long long wait_ns;
  int fail_phase;
  // multi-token prompt path
  bool pf_ok;
  bool sk_ok;  // the skinny projections fit (verify chunks and prompts of <= 8 tokens)
  struct LayerMaps {
    CUtensorMap in_proj, out, q, k, v, gate, up, down;
  } maps[MK_MAX_LAYERS];
  CUtensorMap map_xn, map_a16_dn, map_a16_mlp, map_a16_att, map_embed;
};

namespace {

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MK_OK;
  cudaGetLastError();
  return MK_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int read_device_error(mk_engine* e) {
  int err = 0;
  if (cudaMemcpy(&err, e->ws + e->lay.err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  return err;
}

int launch_decode(mk_engine* e, int pos, int st_in, int st_out, int token, int tok_src,
                  float* logits, int32_t* tok_out) {
  mk::StepArgs a;
  a.m = e->hm;
  a.pos = pos;
  a.token = token;
  a.tok_src = tok_src;
  a.amax_in = e->amax_toggle;
  a.amax_out = e->amax_toggle ^ 1;
  a.st_in = st_in;
  a.st_out = st_out;
  a.logits = logits ? logits : reinterpret_cast<float*>(e->ws + e->lay.logits);
  a.tok_out = tok_out;
  a.hidden = reinterpret_cast<float*>(e->ws + e->lay.hidden);
  // the sequence number names the launch in exchange tags, and its parity
  // selects the set of split-K sum words (consecutive launches alternate)
  uint32_t seq = e->seq + 1;
  if (seq >= (1u << 23)) seq = (seq & 1u) ? 1u : 2u;
  a.seq = seq;
  a.fail_phase = e->fail_phase;
  a.wait_ns = e->wait_ns;
  void* args[] = {&a};
  cudaError_t err = cudaLaunchCooperativeKernel(e->var->fn, dim3(e->ncta), dim3(mk::NTHR), args,
                                                e->var->smem, e->stream);
  if (err != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_LAUNCH;
  }
  e->seq = seq;
  e->fail_phase = -1;
  e->amax_toggle ^= 1;
  e->amax_valid = true;
  e->launches += 1;
  return MK_OK;
}

// One decode launch at the current position that advances the state: it
// reads the current state buffer and writes the next one in the ring.
int replay_pending(mk_engine* e);

int decode_advance(mk_engine* e, int token, int tok_src, float* logits, int32_t* tok_out) {
  const int rp = replay_pending(e);
  if (rp != MK_OK) return rp;
  const int nxt = (e->cur_buf + 1) % mk::kStateBufs;
  const int rc = launch_decode(e, e->pos, e->cur_buf, nxt, token, tok_src, logits, tok_out);
  if (rc == MK_OK) {
    e->cur_buf = nxt;
    e->pos += 1;
  }
  return rc;
}

// One tensor-core GEMM launch.  For a chunk of at most one token tile with
// few output tiles (verify), K is split over gridDim.z so every SM streams
// weights; the partial sums are added atomically, so a non-accumulating
// output is zeroed first.
int launch_gemm(mk_engine* e, const CUtensorMap& tw, const CUtensorMap& tx, float* c, int ldc,
                int n_out, int T, int K, int accumulate) {
  const int tiles = ((n_out + mk::pf::BM - 1) / mk::pf::BM) * ((T + mk::pf::BN - 1) / mk::pf::BN);
  int ks = T <= mk::pf::BN || tiles < kSplitMaxTiles ? (e->ncta + tiles - 1) / tiles : 1;
  if (ks > K / mk::pf::BK) ks = K / mk::pf::BK;
  if (ks < 1) ks = 1;
  if (ks > 1 && T > mk::pf::BN) {
    // a prompt chunk: the ranges' sums go to partial buffers and are added
    // in a fixed order by a second kernel (deterministic, no atomics)
    mk::pf::GemmArgs g;
    g.tw = tw;
    g.tx = tx;
    g.c = c;
    g.ldc = ldc;
    g.n_out = n_out;
    g.T = T;
    g.K = K;
    g.accumulate = accumulate;
    g.x_lo_row = e->lay.tmax;
    g.k_split = ks;
    g.err = e->hm.err;
    g.wait_ns = e->wait_ns;
    float* part = reinterpret_cast<float*>(e->ws + e->lay.pf_part);
    const dim3 grid((n_out + mk::pf::BM - 1) / mk::pf::BM, (T + mk::pf::BN - 1) / mk::pf::BN, ks);
    mk::pf::gemm_tc_partial<<<grid, mk::pf::GEMM_THREADS, mk::pf::GEMM_SMEM, e->stream>>>(g, part);
    const size_t n = size_t(T) * n_out;
    const int rb = int((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    mk::pf::splitk_reduce_ld_kernel<<<rb, 256, 0, e->stream>>>(part, ks, T, n_out, c, ldc,
                                                               accumulate);
    e->launches += 2;
    return cuda_status(cudaGetLastError());
  }
  if (ks > 1 && !accumulate) {
    const cudaError_t r =
        cudaMemset2DAsync(c, size_t(ldc) * 4, 0, size_t(n_out) * 4, T, e->stream);
    if (r != cudaSuccess) return cuda_status(r);
  }
  mk::pf::GemmArgs g;
  g.tw = tw;
  g.tx = tx;
  g.c = c;
  g.ldc = ldc;
  g.n_out = n_out;
  g.T = T;
  g.K = K;
  g.accumulate = accumulate;
  g.x_lo_row = e->lay.tmax;
  g.k_split = ks;
  g.err = e->hm.err;
  g.wait_ns = e->wait_ns;
  const dim3 grid((n_out + mk::pf::BM - 1) / mk::pf::BM, (T + mk::pf::BN - 1) / mk::pf::BN, ks);
  mk::pf::gemm_tc<<<grid, mk::pf::GEMM_THREADS, mk::pf::GEMM_SMEM, e->stream>>>(g);
  e->launches += 1;
  return cuda_status(cudaGetLastError());
}

// A launch that may start while the kernel before it in the stream is
// still running (programmatic stream serialisation); the kernel calls
// griddep_wait() before it reads what that kernel writes.
template <typename... KArgs, typename... Act>
int launch_pdl(mk_engine* e, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
               Act&&... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = e->stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  const cudaError_t r = cudaLaunchKernelEx(&lc, kern, std::forward<Act>(args)...);
  e->launches += 1;
  return cuda_status(r);
}

// The chunk attention instantiation for qt (the query rows rounded up to 8).
template <int HD>
int launch_attn_chunk(mk_engine* e, int qt, dim3 grid, dim3 block, const mk::vf::AttArgs& aa) {
  switch (qt) {
    case 8: return launch_pdl(e, mk::vf::attn_chunk_kernel<HD, 8>, grid, block, mk::vf::att_smem<HD, 8>(), aa);
    case 16: return launch_pdl(e, mk::vf::attn_chunk_kernel<HD, 16>, grid, block, mk::vf::att_smem<HD, 16>(), aa);
    case 24: return launch_pdl(e, mk::vf::attn_chunk_kernel<HD, 24>, grid, block, mk::vf::att_smem<HD, 24>(), aa);
    default: return launch_pdl(e, mk::vf::attn_chunk_kernel<HD, 32>, grid, block, mk::vf::att_smem<HD, 32>(), aa);
  }
}

template <int HD>
bool attn_chunk_attrs() {
  return cudaFuncSetAttribute(mk::vf::attn_chunk_kernel<HD, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(mk::vf::att_smem<HD, 8>())) == cudaSuccess &&
         cudaFuncSetAttribute(mk::vf::attn_chunk_kernel<HD, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(mk::vf::att_smem<HD, 16>())) == cudaSuccess &&
         cudaFuncSetAttribute(mk::vf::attn_chunk_kernel<HD, 24>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(mk::vf::att_smem<HD, 24>())) == cudaSuccess &&
         cudaFuncSetAttribute(mk::vf::attn_chunk_kernel<HD, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(mk::vf::att_smem<HD, 32>())) == cudaSuccess;
}

// One skinny projection (a chunk of T <= 8 tokens): grid of at most two
// CTAs per SM over the output's row blocks, launched so that it may start
// (and stream its first weights) while the kernel before it finishes.
int launch_skinny(mk_engine* e, mk::sk::Args a) {
  a.kw = mk::sk::pick_kw(a.K);
  a.err = e->hm.err;
  a.wait_ns = e->wait_ns;
  const int rpb = (mk::sk::WARPS / a.kw) * mk::sk::RW;
  const int lpb = a.pair ? rpb / 2 : rpb;
  const int nblk = (a.N + lpb - 1) / lpb;
  const dim3 grid(nblk < mk::sk::MAX_CTAS ? nblk : mk::sk::MAX_CTAS), block(mk::sk::THREADS);
  const size_t smem = mk::sk::smem_bytes(a.mode, a.T, a.K, a.dv);
  switch (a.T) {
    case 1: return launch_pdl(e, mk::sk::skinny_gemv_kernel<1>, grid, block, smem, a);
    case 2: return launch_pdl(e, mk::sk::skinny_gemv_kernel<2>, grid, block, smem, a);
    case 3: return launch_pdl(e, mk::sk::skinny_gemv_kernel<3>, grid, block, smem, a);
    case 4: return launch_pdl(e, mk::sk::skinny_gemv_kernel<4>, grid, block, smem, a);
    case 5: return launch_pdl(e, mk::sk::skinny_gemv_kernel<5>, grid, block, smem, a);
    case 6: return launch_pdl(e, mk::sk::skinny_gemv_kernel<6>, grid, block, smem, a);
    case 7: return launch_pdl(e, mk::sk::skinny_gemv_kernel<7>, grid, block, smem, a);
    case 8: return launch_pdl(e, mk::sk::skinny_gemv_kernel<8>, grid, block, smem, a);
  }
  return MK_ERR_ARG;
}

// Largest dynamic shared memory of every skinny instantiation.
bool skinny_attrs(size_t smem) {
  const void* fns[8] = {
      reinterpret_cast<const void*>(mk::sk::skinny_gemv_kernel<1>),
      reinterpret_cast<const void*>(mk::sk::skinny_gemv_kernel<2>),
      reinterpret_cast<const void*>(mk::sk::skinny_gemv_kernel<3>),
      reinterpret_cast<const void*>(mk::sk::skinny_gemv_kernel<4>),
      reinterpret_cast<const void*>(mk::sk::skinny_gemv_kernel<5>),
      reinterpret_cast<const void*>(mk::sk::skinny_gemv_kernel<6>),
      reinterpret_cast<const void*>(mk::sk::skinny_gemv_kernel<7>),
      reinterpret_cast<const void*>(mk::sk::skinny_gemv_kernel<8>)};
  for (const void* f : fns)
    if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
        cudaSuccess)
      return false;
  return true;
}

// Record set `sel` of DeltaNet layer `sub`.
mk::vf::Log vlog(mk_engine* e, int sel, int sub) {
  const Layout& L = e->lay;
  const mk::DevModel& m = e->hm;
  const size_t V = mk::kMaxVerify;
  mk::vf::Log g;
  g.k = reinterpret_cast<float*>(e->ws + L.vlog_k[sel]) + size_t(sub) * V * m.nh * m.dk;
  g.v = reinterpret_cast<float*>(e->ws + L.vlog_v[sel]) + size_t(sub) * V * m.nh * m.dv;
  g.ab = reinterpret_cast<float2*>(e->ws + L.vlog_ab[sel]) + size_t(sub) * V * m.nh;
  g.u = reinterpret_cast<float*>(e->ws + L.vlog_u[sel]) + size_t(sub) * V * m.ch;
  return g;
}

// What a verify chunk replays first (R records of set rsel, the replayed
// state going to buffer nb) and where it writes its own records (set wsel).
struct VerifyPlan {
  int R, rsel, wsel, nb;
};

// Arguments of dn_verify_kernel for DeltaNet layer `sub` (layer 0 plus the
// per-layer strides for a launch over all layers): the state and conv
// history of the current buffer, replayed into buffer nb.
mk::vf::DnArgs dn_args(mk_engine* e, int sub, int R, int rsel, int nb) {
  const mk::DevModel& m = e->hm;
  const size_t soff = size_t(sub) * m.nh * m.dv * m.dk, coff = size_t(sub) * m.ch;
  const size_t V = mk::kMaxVerify;
  mk::vf::DnArgs a{};
  a.S_in = m.dn_state[e->cur_buf] + soff;
  a.S_out = m.dn_state[nb] + soff;
  a.conv_in = reinterpret_cast<const float4*>(m.conv_state[e->cur_buf]) + coff;
  a.conv_out = reinterpret_cast<float4*>(m.conv_state[nb]) + coff;
  a.rlog = vlog(e, rsel, sub);
  a.R = R;
  a.s_stride = size_t(m.nh) * m.dv * m.dk;
  a.c_stride = size_t(m.ch);
  a.lk_stride = V * m.nh * m.dk;
  a.lab_stride = V * m.nh;
  a.lu_stride = V * m.ch;
  a.nh = m.nh;
  a.ch = m.ch;
  return a;
}

// A verify chunk (a.T > 0) may start while the kernel before it finishes and
// runs the CTAs of each head as one cluster when it applies the gated norm;
// a replay (a.T == 0) is a plain launch over all layers.
int launch_dn_verify(mk_engine* e, const mk::vf::DnArgs& a, dim3 grid) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = dim3(mk::vf::THREADS);
  lc.stream = e->stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = 1;
  at[1].val.clusterDim.y = grid.y;
  at[1].val.clusterDim.z = 1;
  lc.attrs = at;
  lc.numAttrs = a.T == 0 ? 0 : a.out_norm ? 2 : 1;
  const cudaError_t r = e->hm.dk == 128 ? cudaLaunchKernelEx(&lc, mk::vf::dn_verify_kernel<128>, a)
                                        : cudaLaunchKernelEx(&lc, mk::vf::dn_verify_kernel<64>, a);
  e->launches += 1;
  return cuda_status(r);
}

// Apply the accepted records of the last verify to the state (into the next
// state buffer) before a call that reads the state in another way.
int replay_pending(mk_engine* e) {
  if (e->replay_n == 0) return MK_OK;
  const mk::DevModel& m = e->hm;
  const int nb = (e->cur_buf + 1) % mk::kStateBufs;
  if (m.n_dn > 0) {
    const mk::vf::DnArgs a = dn_args(e, 0, e->replay_n, e->replay_sel, nb);
    const int rc = launch_dn_verify(e, a, dim3(m.nh, m.dv / mk::vf::BR, m.n_dn));
    if (rc != MK_OK) return rc;
  }
  e->cur_buf = nb;
  e->replay_n = 0;
  return MK_OK;
}

// The stack over T positions starting at e->pos through the chunk kernels.
// Prompt chunk (vp == nullptr): the state is updated in place and the
// position advances.  Verify chunk: the pending records are replayed into
// buffer vp->nb (when vp->R > 0), the chunk writes its records to set
// vp->wsel and no state, the position does not move, and logits_out
// [T][vocab] receives every position's logits.
int run_chunk(mk_engine* e, const int32_t* tokens_host, int T, const VerifyPlan* vp,
              float* logits_out) {
  using namespace mk::pf;
  const mk_config& c = e->cfg;
  const Layout& L = e->lay;
  const mk::DevModel& m = e->hm;
  char* ws = e->ws;
  cudaStream_t st = e->stream;
  const int H = c.hidden, pw = L.pw, aw = L.aw, pos0 = e->pos;
  const size_t lo_x = size_t(L.tmax) * H, lo_a = size_t(L.tmax) * aw;  // lo operand offsets
  const int nh = c.dn_heads, dk = c.dn_dk, dv = c.dn_dv, I = c.mlp;
  const int nq = c.q_heads, nkv = c.kv_heads, hd = c.head_dim;
  int32_t* tok = reinterpret_cast<int32_t*>(ws + L.pf_tok);
  float* X = reinterpret_cast<float*>(ws + L.pf_x);
  uint16_t* Xn = reinterpret_cast<uint16_t*>(ws + L.pf_xn);
  float* P = reinterpret_cast<float*>(ws + L.pf_p);
  float* O = reinterpret_cast<float*>(ws + L.pf_o);
  uint16_t* A16 = reinterpret_cast<uint16_t*>(ws + L.pf_a16);
  float* QK = reinterpret_cast<float*>(ws + L.pf_qk);
  float4* BAK = reinterpret_cast<float4*>(ws + L.pf_bak);
  // at most 8 tokens: every projection is one weight-streaming pass with its
  // operand's producer (RMSNorm, SwiGLU, gated norm) fused into its prologue
  const bool sk = T <= mk::sk::TMAX && e->sk_ok;
  // fp32 view of the bf16 operand buffer: the attention output and SiLU(gate)
  // * up of a skinny chunk, [T][aw]
  float* Af = reinterpret_cast<float*>(A16);
  auto sk_norm = [&](const uint16_t* W0, const uint16_t* W1, int N, const uint16_t* gain,
                     float* C, int ldc) {
    mk::sk::Args a{};
    a.W0 = W0;
    a.W1 = W1;
    a.pair = W1 != nullptr;
    a.N = N;
    a.K = H;
    a.T = T;
    a.mode = mk::sk::X_NORM;
    a.X = X;
    a.ldx = H;
    a.gain = gain;
    a.eps = c.rms_eps;
    a.C = C;
    a.ldc = ldc;
    return launch_skinny(e, a);
  };
  if (!vp) {
    const int rp = replay_pending(e);
    if (rp != MK_OK) return rp;
  }
  cudaError_t r = cudaMemcpyAsync(tok, tokens_host, size_t(T) * 4, cudaMemcpyHostToDevice, st);
  if (r != cudaSuccess) return cuda_status(r);
  embed_kernel<<<T, ROW_THREADS, 0, st>>>(tok, m.embed, X, H);
  e->launches += 1;
  int rc = MK_OK;
  for (int l = 0; l < c.n_layers && rc == MK_OK; ++l) {
    const mk::DevLayer& D = m.layers[l];
    const mk_engine::LayerMaps& mp = e->maps[l];
    if (!sk) rmsnorm_bf16_kernel<<<T, ROW_THREADS, 0, st>>>(X, D.attn_norm, Xn, H, c.rms_eps, lo_x);
    if (!D.is_attn) {
      rc = sk ? sk_norm(D.in_proj, nullptr, m.rin, D.attn_norm, P, pw)
              : launch_gemm(e, mp.in_proj, e->map_xn, P, pw, m.rin, T, H, 0);
      if (vp) {
        // verify: replay, conv, gates and recurrence in one kernel, which
        // records the chunk's positions instead of writing states
        mk::vf::DnArgs a = dn_args(e, D.sub, vp->R, vp->rsel, vp->nb);
        a.wlog = vlog(e, vp->wsel, D.sub);
        a.P = P;
        a.ldp = pw;
        a.conv_w = D.conv_w;
        a.A_log = D.A_log;
        a.dt_bias = D.dt_bias;
        a.O = O;
        a.ldo = nh * dv;
        a.out_norm = sk ? D.out_norm : nullptr;  // else the gated norm kernel below
        a.eps = c.rms_eps;
        a.zcol = m.ch;
        a.T = T;
        if (rc == MK_OK) rc = launch_dn_verify(e, a, dim3(nh, dv / mk::vf::BR));
      } else {
        float4* cst = reinterpret_cast<float4*>(m.conv_state[e->cur_buf]) + size_t(D.sub) * m.ch;
        float* Cv = reinterpret_cast<float*>(ws + L.pf_c);
        conv_kernel<<<dim3((m.ch + 255) / 256, T), 256, 0, st>>>(P, pw, cst, D.conv_w, m.ch, Cv,
                                                                m.ch);
        conv_state_kernel<<<(m.ch + 255) / 256, 256, 0, st>>>(P, pw, cst, m.ch, T);
        dn_prep_kernel<<<dim3(T, nh), dk, 0, st>>>(Cv, m.ch, P, pw, nh, dk, m.ch, dv, D.A_log,
                                                   D.dt_bias, QK, BAK, T);
        float* S = m.dn_state[e->cur_buf] + size_t(D.sub) * nh * dv * dk;
        const int vcol = 2 * nh * dk;
        // the chunkwise-parallel form (independent per chunk of 64
        // positions, then one pass over the chunks)
        float* prep = reinterpret_cast<float*>(ws + L.pf_chunk);
        const dim3 pg((T + mk::ck::C - 1) / mk::ck::C, nh), sg(dv / mk::ck::SCAN_ROWS, nh);
        if (dk == 128) {
          mk::ck::chunk_prep_kernel<128><<<pg, mk::ck::PREP_THREADS, mk::ck::prep_smem<128>(), st>>>(
              QK, BAK, Cv + vcol, size_t(m.ch), size_t(dk), T, prep);
          mk::ck::chunk_scan_kernel<128><<<sg, mk::ck::SCAN_THREADS, mk::ck::scan_smem<128>(), st>>>(
              S, prep, T, O, size_t(nh) * dv, size_t(dv));
        } else {
          mk::ck::chunk_prep_kernel<64><<<pg, mk::ck::PREP_THREADS, mk::ck::prep_smem<64>(), st>>>(
              QK, BAK, Cv + vcol, size_t(m.ch), size_t(dk), T, prep);
          mk::ck::chunk_scan_kernel<64><<<sg, mk::ck::SCAN_THREADS, mk::ck::scan_smem<64>(), st>>>(
              S, prep, T, O, size_t(nh) * dv, size_t(dv));
        }
        e->launches += 5;  // conv, its state, gates, chunk prep and scan
      }
      if (sk) {
        mk::sk::Args a{};
        a.W0 = D.out_proj;
        a.N = H;
        a.K = nh * dv;
        a.T = T;
        // verify: O holds the gated-normed readout already
        a.mode = vp ? mk::sk::X_COPY : mk::sk::X_GATED;
        a.X = O;
        a.ldx = nh * dv;
        a.X2 = P + m.ch;  // z
        a.ldx2 = pw;
        a.dv = dv;
        a.gain = D.out_norm;
        a.eps = c.rms_eps;
        a.C = X;
        a.ldc = H;
        a.accumulate = 1;
        if (rc == MK_OK) rc = launch_skinny(e, a);
      } else {
        gated_norm_kernel<<<dim3(T, nh), dv, 0, st>>>(O, nh * dv, P, pw, m.ch, D.out_norm, A16,
                                                      aw, c.rms_eps, lo_a);
        if (rc == MK_OK) rc = launch_gemm(e, mp.out, e->map_a16_dn, X, H, H, T, nh * dv, 1);
      }
    } else {
      if (sk) {
        rc = sk_norm(D.w_qkv, nullptr, (nq + 2 * nkv) * hd, D.attn_norm, P, pw);
      } else {
        rc = launch_gemm(e, mp.q, e->map_xn, P, pw, nq * hd, T, H, 0);
        if (rc == MK_OK) rc = launch_gemm(e, mp.k, e->map_xn, P + nq * hd, pw, nkv * hd, T, H, 0);
        if (rc == MK_OK)
          rc = launch_gemm(e, mp.v, e->map_xn, P + (nq + nkv) * hd, pw, nkv * hd, T, H, 0);
      }
      const size_t kvo = size_t(D.sub) * nkv * c.max_ctx * hd;
      if (sk && (nq / nkv) * T <= mk::vf::ATT_QMAX) {
        // rope + KV append, the chunk attention over key ranges and their
        // merge, each starting while the kernel before it finishes
        if (rc == MK_OK)
          rc = launch_pdl(e, rope_kv_kernel, dim3(T, nq + nkv), dim3(hd / 2), 0, P, pw, nq, nkv,
                          hd, m.kc + kvo, m.vc + kvo, c.max_ctx, pos0, c.rope_theta);
        mk::vf::AttArgs aa{};
        aa.P = P;
        aa.ldp = pw;
        aa.kc = m.kc + kvo;
        aa.vc = m.vc + kvo;
        aa.max_ctx = c.max_ctx;
        aa.nq = nq;
        aa.nkv = nkv;
        aa.pos0 = pos0;
        aa.T = T;
        aa.nsplit = (pos0 + T + mk::vf::ATT_L - 1) / mk::vf::ATT_L;
        aa.part = reinterpret_cast<float*>(ws + L.pf_att);
        aa.out = Af;
        aa.ldo = aw;
        const dim3 ag(aa.nsplit, nkv), mg(nq, T), tb(mk::vf::ATT_THREADS);
        const int qt = ((nq / nkv) * T + 7) / 8 * 8;
        if (rc == MK_OK) {
          if (hd == 256)
            rc = launch_attn_chunk<256>(e, qt, ag, tb, aa);
          else if (hd == 128)
            rc = launch_attn_chunk<128>(e, qt, ag, tb, aa);
          else
            rc = launch_attn_chunk<64>(e, qt, ag, tb, aa);
        }
        if (rc == MK_OK) {
          if (hd == 256)
            rc = launch_pdl(e, mk::vf::attn_chunk_merge<256>, mg, tb, 0, aa);
          else if (hd == 128)
            rc = launch_pdl(e, mk::vf::attn_chunk_merge<128>, mg, tb, 0, aa);
          else
            rc = launch_pdl(e, mk::vf::attn_chunk_merge<64>, mg, tb, 0, aa);
        }
      } else if (T <= mk::kMaxVerify) {
        rope_kv_kernel<<<dim3(T, nq + nkv), hd / 2, 0, st>>>(P, pw, nq, nkv, hd, m.kc + kvo,
                                                             m.vc + kvo, c.max_ctx, pos0,
                                                             c.rope_theta);
        // few queries: split the keys too, then merge the ranges
        float* part = reinterpret_cast<float*>(ws + L.pf_att);
        const int nsplit = (pos0 + T + ATT_SPLIT_LEN - 1) / ATT_SPLIT_LEN;
        const dim3 sg((nsplit + ATT_SPLIT_WARPS - 1) / ATT_SPLIT_WARPS, nq, T);
        const dim3 mg(nq, T);
        if (hd == 256) {
          attn_split_kernel<256><<<sg, ATT_SPLIT_WARPS * 32, 0, st>>>(
              P, pw, m.kc + kvo, m.vc + kvo, c.max_ctx, nq, nkv, pos0, nsplit, part);
          attn_merge_kernel<256><<<mg, 256, 0, st>>>(part, nq, nsplit, A16, aw, lo_a,
                                                      sk ? Af : nullptr);
        } else if (hd == 128) {
          attn_split_kernel<128><<<sg, ATT_SPLIT_WARPS * 32, 0, st>>>(
              P, pw, m.kc + kvo, m.vc + kvo, c.max_ctx, nq, nkv, pos0, nsplit, part);
          attn_merge_kernel<128><<<mg, 128, 0, st>>>(part, nq, nsplit, A16, aw, lo_a,
                                                      sk ? Af : nullptr);
        } else {
          attn_split_kernel<64><<<sg, ATT_SPLIT_WARPS * 32, 0, st>>>(
              P, pw, m.kc + kvo, m.vc + kvo, c.max_ctx, nq, nkv, pos0, nsplit, part);
          attn_merge_kernel<64><<<mg, 64, 0, st>>>(part, nq, nsplit, A16, aw, lo_a,
                                                      sk ? Af : nullptr);
        }
        e->launches += 3;  // rope, key ranges, merge
      } else {
        rope_kv_kernel<<<dim3(T, nq + nkv), hd / 2, 0, st>>>(P, pw, nq, nkv, hd, m.kc + kvo,
                                                             m.vc + kvo, c.max_ctx, pos0,
                                                             c.rope_theta);
        e->launches += 2;  // rope, attention
        const dim3 agrid((T + 7) / 8, nq);
        mk::vf::PromptAttArgs pa{};
        pa.P = P;
        pa.ldp = pw;
        pa.kc = m.kc + kvo;
        pa.vc = m.vc + kvo;
        pa.max_ctx = c.max_ctx;
        pa.nq = nq;
        pa.nkv = nkv;
        pa.pos0 = pos0;
        pa.T = T;
        pa.Ob = A16;
        pa.ldo = aw;
        pa.lo = lo_a;
        const dim3 pg((T + mk::vf::PR_POS - 1) / mk::vf::PR_POS, nkv), pb(mk::vf::ATT_THREADS);
        // flash-style tiles when a block's query rows fit one CTA
        const bool flash = e->sk_ok && (nq / nkv) * mk::vf::PR_POS <= mk::vf::ATT_QMAX;
        if (flash && hd == 256)
          mk::vf::attn_prompt_kernel<256><<<pg, pb, mk::vf::prompt_att_smem<256>(), st>>>(pa);
        else if (flash && hd == 128)
          mk::vf::attn_prompt_kernel<128><<<pg, pb, mk::vf::prompt_att_smem<128>(), st>>>(pa);
        else if (flash)
          mk::vf::attn_prompt_kernel<64><<<pg, pb, mk::vf::prompt_att_smem<64>(), st>>>(pa);
        else if (hd == 256)
          attn_prefill_kernel<256><<<agrid, 256, 0, st>>>(P, pw, m.kc + kvo, m.vc + kvo,
                                                          c.max_ctx, nq, nkv, pos0, T, A16, aw,
                                                          lo_a);
        else if (hd == 128)
          attn_prefill_kernel<128><<<agrid, 256, 0, st>>>(P, pw, m.kc + kvo, m.vc + kvo,
                                                          c.max_ctx, nq, nkv, pos0, T, A16, aw,
                                                          lo_a);
        else
          attn_prefill_kernel<64><<<agrid, 256, 0, st>>>(P, pw, m.kc + kvo, m.vc + kvo,
                                                         c.max_ctx, nq, nkv, pos0, T, A16, aw,
                                                         lo_a);
      }
      if (sk) {
        mk::sk::Args a{};
        a.W0 = D.w_o;
        a.N = H;
        a.K = nq * hd;
        a.T = T;
        a.mode = mk::sk::X_COPY;
        a.X = Af;
        a.ldx = aw;
        a.C = X;
        a.ldc = H;
        a.accumulate = 1;
        if (rc == MK_OK) rc = launch_skinny(e, a);
      } else if (rc == MK_OK) {
        rc = launch_gemm(e, mp.out, e->map_a16_att, X, H, H, T, nq * hd, 1);
      }
    }
    if (sk) {
      if (rc == MK_OK) rc = sk_norm(D.w_gate, D.w_up, I, D.mlp_norm, Af, aw);
      mk::sk::Args a{};
      a.W0 = D.w_down;
      a.N = H;
      a.K = I;
      a.T = T;
      a.mode = mk::sk::X_COPY;
      a.X = Af;
      a.ldx = aw;
      a.C = X;
      a.ldc = H;
      a.accumulate = 1;
      if (rc == MK_OK) rc = launch_skinny(e, a);

    } else {
      rmsnorm_bf16_kernel<<<T, ROW_THREADS, 0, st>>>(X, D.mlp_norm, Xn, H, c.rms_eps, lo_x);
      if (rc == MK_OK) rc = launch_gemm(e, mp.gate, e->map_xn, P, pw, I, T, H, 0);
      if (rc == MK_OK) rc = launch_gemm(e, mp.up, e->map_xn, P + I, pw, I, T, H, 0);
      swiglu_kernel<<<dim3((I + 255) / 256, T), 256, 0, st>>>(P, pw, I, A16, aw, lo_a);
      if (rc == MK_OK) rc = launch_gemm(e, mp.down, e->map_a16_mlp, X, H, H, T, I, 1);
      e->launches += D.is_attn ? 3 : 4;  // norms, SwiGLU (and the gated norm)
    }
  }
  if (rc != MK_OK) return rc;
  if (logits_out) {
    // final norm and the tied LM head for every position of the chunk
    if (sk) {
      rc = sk_norm(m.embed, nullptr, c.vocab, m.final_norm, logits_out, c.vocab);
    } else {
      rmsnorm_bf16_kernel<<<T, ROW_THREADS, 0, st>>>(X, m.final_norm, Xn, H, c.rms_eps, lo_x);
      e->launches += 1;
      rc = launch_gemm(e, e->map_embed, e->map_xn, logits_out, c.vocab, c.vocab, T, H, 0);
    }
    if (rc != MK_OK) return rc;
  }
  r = cudaGetLastError();
  if (r != cudaSuccess) return cuda_status(r);
  if (!vp) e->pos += T;
  return MK_OK;
}

}  // namespace

extern "C" {

size_t mk_workspace_bytes(const mk_config* cfg) {
  if (!basic_valid(cfg)) return 0;
  return make_layout(*cfg).total;
}

int mk_create(const mk_config* cfg, const mk_weights* w, void* workspace, size_t ws_bytes,
              void* cuda_stream, mk_engine** out) {
  if (!out) return MK_ERR_ARG;
  *out = nullptr;
  if (!basic_valid(cfg) || !w || !workspace || !w->embed || !w->final_norm || !w->layers)
    return MK_ERR_ARG;
  const mk_config& c = *cfg;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MK_ERR_ARG;
  Layout lay = make_layout(c);
  if (ws_bytes < lay.total) return MK_ERR_ARG;

  // shapes the kernels implement
  const int G = c.q_heads / c.kv_heads;
  const Variant* var = find_variant(c.dn_dk, c.head_dim, G);
  if (!var || c.dn_dk != c.dn_dv || c.conv_k != 4) return MK_ERR_UNSUPPORTED;
  if (c.hidden % 256 || c.hidden > 2048 || c.mlp % 8 || c.mlp > 4096) return MK_ERR_UNSUPPORTED;
  if (c.dn_heads * c.dn_dv > 4096 || c.q_heads * c.head_dim > 4096) return MK_ERR_UNSUPPORTED;
  if (2 * c.mlp > mk::SLOT || c.head_dim * 2 * 2 > mk::SLOT) return MK_ERR_UNSUPPORTED;
  if (c.dn_heads * c.dn_dv > 2048 || c.mlp > mk::UNION_FLOATS) return MK_ERR_UNSUPPORTED;

  // weights: present and 16-byte aligned
  if (!aligned16(w->embed) || !aligned16(w->final_norm)) return MK_ERR_ARG;
  for (int l = 0; l < c.n_layers; ++l) {
    const mk_layer_weights& L = w->layers[l];
    const void* common[] = {L.attn_norm, L.mlp_norm, L.w_gate, L.w_up, L.w_down};
    for (const void* p : common)
      if (!p || !aligned16(p)) return MK_ERR_ARG;
    if (c.layer_is_attn[l]) {
      const void* ps[] = {L.w_q, L.w_k, L.w_v, L.w_o};
      for (const void* p : ps)
        if (!p || !aligned16(p)) return MK_ERR_ARG;
    } else {
      const void* ps[] = {L.in_proj, L.conv_w, L.A_log, L.dt_bias, L.out_norm, L.out_proj};
      for (const void* p : ps)
        if (!p || !aligned16(p)) return MK_ERR_ARG;
    }
  }

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MK_ERR_CUDA;
  int nsm = 0, coop = 0;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
  if (!coop || nsm <= 0) return MK_ERR_LAUNCH;
  const int ncta = nsm < mk::kMaxCtas ? nsm : mk::kMaxCtas;
  // the decode kernel keeps its per-launch schedule in shared memory
  if (c.n_layers * mk::PHASES_PER_LAYER + 1 > mk::MAX_PHASES) return MK_ERR_UNSUPPORTED;
  // decode groups: one per DeltaNet head, gs CTAs each
  const int ng = c.dn_heads, gs = ncta / ng;
  if (gs < 1 || ng > 255) return MK_ERR_UNSUPPORTED;
  if ((c.q_heads * c.head_dim) % ng || c.mlp % ng) return MK_ERR_UNSUPPORTED;
  const int kb_att = c.q_heads * c.head_dim / ng, kb_mlp = c.mlp / ng;
  const int rin_h = 2 * c.dn_dk + 2 * c.dn_dv + 2;
  // K blocks of the split-K rows: 16-byte rows; the attention block fits
  // the merge staging; the conv staging holds a CTA's in-projection rows
  if (kb_att % 8 || kb_mlp % 8 || kb_att > 256 || kb_att > mk::MERGE_STAGE)
    return MK_ERR_UNSUPPORTED;
  if ((rin_h + gs - 1) / gs > mk::CONV_ROWS_MAX) return MK_ERR_UNSUPPORTED;
  {
    // attention scratch of the split phase, and of the merge: staged values,
    // (m, l) and weights of every split for the q heads one block touches
    const int smax = ncta / c.kv_heads;
    const int att = 2 * G * c.head_dim + 2 * c.head_dim + mk::NCW * G * 2;
    const int nhb = (kb_att + c.head_dim - 1) / c.head_dim + 1;
    if (att > mk::UNION_FLOATS || nhb > mk::MERGE_HEADS_MAX ||
        2 * smax * nhb > mk::MERGE_ML_MAX ||
        mk::MERGE_STAGE + 3 * smax * nhb > mk::UNION_FLOATS - 256)
      return MK_ERR_UNSUPPORTED;
  }
  // the kernel's balanced splits multiply in 32 bits
  if (uint64_t(c.max_ctx + 1) * ncta >= (uint64_t(1) << 32) ||
      uint64_t(c.vocab) * ncta >= (uint64_t(1) << 32))
    return MK_ERR_UNSUPPORTED;
  // one DeltaNet head's state is one ring chunk of the state phase
  if (size_t(c.dn_dv) * c.dn_dk * 4 > size_t(mk::SLOT)) return MK_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(var->fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(var->smem)) != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_LAUNCH;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, var->fn, mk::NTHR, var->smem) !=
          cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    return MK_ERR_LAUNCH;
  }
  mk_engine* e = new (std::nothrow) mk_engine();
  if (!e) return MK_ERR_ARG;
  e->cfg = c;
  e->device = dev;
  e->stream = static_cast<cudaStream_t>(cuda_stream);
  e->ws = static_cast<char*>(workspace);
  e->lay = lay;
  e->var = var;
  e->ncta = ncta;
  e->wait_ns = 2000000000LL;
  e->fail_phase = -1;

  DevModel& m = e->hm;
  std::memset(&m, 0, sizeof m);
  m.n_layers = c.n_layers;
  m.n_attn = count_attn(c);
  m.n_dn = c.n_layers - m.n_attn;
  m.H = c.hidden;
  m.V = c.vocab;
  m.I = c.mlp;
  m.nh = c.dn_heads;
  m.dk = c.dn_dk;
  m.dv = c.dn_dv;
  m.ck = c.conv_k;
  m.ch = 2 * c.dn_heads * c.dn_dk + c.dn_heads * c.dn_dv;
  m.rin = m.ch + c.dn_heads * c.dn_dv + 2 * c.dn_heads;
  m.nq = c.q_heads;
  m.nkv = c.kv_heads;
  m.hd = c.head_dim;
  m.max_ctx = c.max_ctx;
  m.max_verify = c.max_verify;
  m.ncta = ncta;
  m.ng = ng;
  m.gs = gs;
  m.rin_h = rin_h;
  m.kb_att = kb_att;
  m.kb_mlp = kb_mlp;
  m.eps = c.rms_eps;
  m.theta = c.rope_theta;
  m.embed = static_cast<const uint16_t*>(w->embed);
  m.final_norm = static_cast<const uint16_t*>(w->final_norm);
  int nd = 0, na = 0;
  for (int l = 0; l < c.n_layers; ++l) {
    const mk_layer_weights& L = w->layers[l];
    mk::DevLayer& D = m.layers[l];
    D.attn_norm = static_cast<const uint16_t*>(L.attn_norm);
    D.in_proj = static_cast<const uint16_t*>(L.in_proj);
    D.conv_w = static_cast<const uint16_t*>(L.conv_w);
    D.A_log = L.A_log;
    D.dt_bias = L.dt_bias;
    D.out_norm = static_cast<const uint16_t*>(L.out_norm);
    D.out_proj = static_cast<const uint16_t*>(L.out_proj);
    D.w_q = static_cast<const uint16_t*>(L.w_q);
    D.w_k = static_cast<const uint16_t*>(L.w_k);
    D.w_v = static_cast<const uint16_t*>(L.w_v);
    D.w_o = static_cast<const uint16_t*>(L.w_o);
    D.w_qkv = nullptr;
    D.w_in_pk = nullptr;
    D.w_out_blk = nullptr;
    D.w_down_blk = nullptr;
    D.mlp_norm = static_cast<const uint16_t*>(L.mlp_norm);
    D.w_gate = static_cast<const uint16_t*>(L.w_gate);
    D.w_up = static_cast<const uint16_t*>(L.w_up);
    D.w_down = static_cast<const uint16_t*>(L.w_down);
    D.is_attn = c.layer_is_attn[l] ? 1 : 0;
    D.sub = D.is_attn ? na++ : nd++;
  }
  char* ws = e->ws;
  for (int b = 0; b < mk::kStateBufs; ++b) {
    m.dn_state[b] = reinterpret_cast<float*>(ws + lay.dn_state[b]);
    m.conv_state[b] = reinterpret_cast<float*>(ws + lay.conv_state[b]);
  }
  m.kc = reinterpret_cast<uint16_t*>(ws + lay.kc);
  m.vc = reinterpret_cast<uint16_t*>(ws + lay.vc);
  {
    // Weight copies for the decode kernel's partition (made once, on the
    // engine's stream): each attention layer's q, k and v rows as one
    // matrix; each DeltaNet head's in-projection rows q|k|v|z|b|a
    // contiguous; every output projection and MLP down projection split into
    // ng blocks of K columns, block g stored as its own [H][K/ng] matrix.
    cudaStream_t st = e->stream;
    cudaError_t r = cudaSuccess;
    const size_t H2 = size_t(c.hidden) * 2;
    const size_t qb = size_t(c.q_heads) * c.head_dim * H2, kb = size_t(c.kv_heads) * c.head_dim * H2;
    const size_t dkr = size_t(c.dn_dk) * H2, dvr = size_t(c.dn_dv) * H2;
    char* out_dst = ws + lay.w_out_blk;
    for (int l = 0; l < c.n_layers && r == cudaSuccess; ++l) {
      mk::DevLayer& D = m.layers[l];
      // split-K copy of a [H][K] matrix into ng blocks [H][K/ng]
      auto blocks = [&](char* dst, const void* src, int K) {
        const size_t kbytes = size_t(K / ng) * 2;
        for (int g = 0; g < ng && r == cudaSuccess; ++g)
          r = cudaMemcpy2DAsync(dst + size_t(g) * c.hidden * kbytes, kbytes,
                                static_cast<const char*>(src) + size_t(g) * kbytes, size_t(K) * 2,
                                kbytes, size_t(c.hidden), cudaMemcpyDeviceToDevice, st);
      };
      if (D.is_attn) {
        char* dst = ws + lay.wqkv + size_t(D.sub) * (qb + 2 * kb);
        r = cudaMemcpyAsync(dst, D.w_q, qb, cudaMemcpyDeviceToDevice, st);
        if (r == cudaSuccess) r = cudaMemcpyAsync(dst + qb, D.w_k, kb, cudaMemcpyDeviceToDevice, st);
        if (r == cudaSuccess)
          r = cudaMemcpyAsync(dst + qb + kb, D.w_v, kb, cudaMemcpyDeviceToDevice, st);
        D.w_qkv = reinterpret_cast<const uint16_t*>(dst);
        blocks(out_dst, D.w_o, c.q_heads * c.head_dim);
        D.w_out_blk = reinterpret_cast<const uint16_t*>(out_dst);
        out_dst += size_t(c.q_heads) * c.head_dim * H2;
      } else {
        const char* src = reinterpret_cast<const char*>(D.in_proj);
        char* dst = ws + lay.w_in_pk + size_t(D.sub) * c.dn_heads * rin_h * H2;
        D.w_in_pk = reinterpret_cast<const uint16_t*>(dst);
        const size_t ch_rows = 2 * size_t(c.dn_heads) * c.dn_dk + size_t(c.dn_heads) * c.dn_dv;
        for (int h = 0; h < c.dn_heads && r == cudaSuccess; ++h) {
          // rows of head h in the caller's layout [q | k | v | z | b | a]
          const size_t seg_src[6] = {
              size_t(h) * dkr, size_t(c.dn_heads) * dkr + h * dkr,
              2 * size_t(c.dn_heads) * dkr + h * dvr, ch_rows * H2 + h * dvr,
              (ch_rows + size_t(c.dn_heads) * c.dn_dv + h) * H2,
              (ch_rows + size_t(c.dn_heads) * c.dn_dv + c.dn_heads + h) * H2};
          const size_t seg_len[6] = {dkr, dkr, dvr, dvr, H2, H2};
          for (int q = 0; q < 6 && r == cudaSuccess; ++q) {
            r = cudaMemcpyAsync(dst, src + seg_src[q], seg_len[q], cudaMemcpyDeviceToDevice, st);
            dst += seg_len[q];
          }
        }
        blocks(out_dst, D.out_proj, c.dn_heads * c.dn_dv);
        D.w_out_blk = reinterpret_cast<const uint16_t*>(out_dst);
        out_dst += size_t(c.dn_heads) * c.dn_dv * H2;
      }
      char* ddst = ws + lay.w_down_blk + size_t(l) * c.mlp * H2;
      blocks(ddst, D.w_down, c.mlp);
      D.w_down_blk = reinterpret_cast<const uint16_t*>(ddst);
    }
    if (r != cudaSuccess) {
      delete e;
      return cuda_status(r);
    }
  }
  using ull = unsigned long long;
  m.xacc = reinterpret_cast<ull*>(ws + lay.xacc);
  m.grp_inp = reinterpret_cast<ull*>(ws + lay.grp_inp);
  m.grp_h = reinterpret_cast<ull*>(ws + lay.grp_h);
  m.qkv_ll = reinterpret_cast<ull*>(ws + lay.qkv);
  m.part_ll = reinterpret_cast<ull*>(ws + lay.part);
  m.hidden = reinterpret_cast<float*>(ws + lay.hidden);
  m.logits_scratch = reinterpret_cast<float*>(ws + lay.logits);
  m.tickets = reinterpret_cast<unsigned*>(ws + lay.tickets);
  m.err = reinterpret_cast<int*>(ws + lay.err);
  m.amax = reinterpret_cast<unsigned long long*>(ws + lay.amax);
  e->dm = reinterpret_cast<DevModel*>(ws + lay.model);
  if (cudaMemcpyAsync(e->dm, &m, sizeof m, cudaMemcpyHostToDevice, e->stream) != cudaSuccess ||
      cudaStreamSynchronize(e->stream) != cudaSuccess) {
    cudaGetLastError();
    delete e;
    return MK_ERR_CUDA;
  }
  // tensor maps of the prompt path (weights and the chunk's bf16 activations)
  e->pf_ok = cudaFuncSetAttribute(mk::ck::chunk_prep_kernel<128>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(mk::ck::prep_smem<128>())) == cudaSuccess &&
             cudaFuncSetAttribute(mk::ck::chunk_scan_kernel<128>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(mk::ck::scan_smem<128>())) == cudaSuccess &&
             cudaFuncSetAttribute(mk::ck::chunk_prep_kernel<64>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(mk::ck::prep_smem<64>())) == cudaSuccess &&
             cudaFuncSetAttribute(mk::ck::chunk_scan_kernel<64>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(mk::ck::scan_smem<64>())) == cudaSuccess &&
             cudaFuncSetAttribute(mk::pf::gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(mk::pf::GEMM_SMEM)) == cudaSuccess &&
             cudaFuncSetAttribute(mk::pf::gemm_tc_partial,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(mk::pf::GEMM_SMEM)) == cudaSuccess;
  {
    // widest K of a skinny projection: hidden, MLP, DeltaNet readout, attention
    int kmax = c.hidden;
    if (c.mlp > kmax) kmax = c.mlp;
    if (c.dn_heads * c.dn_dv > kmax) kmax = c.dn_heads * c.dn_dv;
    if (c.q_heads * c.head_dim > kmax) kmax = c.q_heads * c.head_dim;
    size_t smem = mk::sk::smem_bytes(mk::sk::X_NORM, mk::sk::TMAX, c.hidden, 0);
    const size_t sg = mk::sk::smem_bytes(mk::sk::X_GATED, mk::sk::TMAX, c.dn_heads * c.dn_dv,
                                         c.dn_dv);
    const size_t sc = mk::sk::smem_bytes(mk::sk::X_COPY, mk::sk::TMAX, kmax, 0);
    if (sg > smem) smem = sg;
    if (sc > smem) smem = sc;
    // bulk-copied operand rows start 16-byte aligned
    const bool rows16 = c.hidden % 128 == 0 && c.hidden <= 4096 && e->lay.pw % 4 == 0 && e->lay.aw % 4 == 0 &&
                        (c.dn_heads * c.dn_dv) % 4 == 0 && e->hm.ch % 4 == 0 && c.mlp % 8 == 0 &&
                        (c.q_heads * c.head_dim) % 8 == 0;
    e->sk_ok = smem <= 227u * 1024u && c.dn_dv % 32 == 0 && rows16 && skinny_attrs(smem) &&
               attn_chunk_attrs<256>() && attn_chunk_attrs<128>() && attn_chunk_attrs<64>() &&
               cudaFuncSetAttribute(mk::vf::attn_prompt_kernel<256>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    int(mk::vf::prompt_att_smem<256>())) == cudaSuccess &&
               cudaFuncSetAttribute(mk::vf::attn_prompt_kernel<128>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    int(mk::vf::prompt_att_smem<128>())) == cudaSuccess &&
               cudaFuncSetAttribute(mk::vf::attn_prompt_kernel<64>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    int(mk::vf::prompt_att_smem<64>())) == cudaSuccess;
  }
  cudaGetLastError();
  {
    const int H = c.hidden, T = lay.tmax;
    const int qd = c.q_heads * c.head_dim, kd = c.kv_heads * c.head_dim;
    const int vd = c.dn_heads * c.dn_dv;
    bool ok = e->pf_ok;
    ok = ok && make_map(&e->map_xn, ws + lay.pf_xn, 2 * T, H, H, mk::pf::BN);
    ok = ok && make_map(&e->map_embed, w->embed, c.vocab, H, H, mk::pf::BM);
    ok = ok && make_map(&e->map_a16_dn, ws + lay.pf_a16, 2 * T, vd, lay.aw, mk::pf::BN);
    ok = ok && make_map(&e->map_a16_mlp, ws + lay.pf_a16, 2 * T, c.mlp, lay.aw, mk::pf::BN);
    ok = ok && make_map(&e->map_a16_att, ws + lay.pf_a16, 2 * T, qd, lay.aw, mk::pf::BN);
    for (int l = 0; l < c.n_layers && ok; ++l) {
      const mk_layer_weights& L = w->layers[l];
      mk_engine::LayerMaps& mp = e->maps[l];
      const int BM = mk::pf::BM;
      ok = make_map(&mp.gate, L.w_gate, c.mlp, H, H, BM) &&
           make_map(&mp.up, L.w_up, c.mlp, H, H, BM) &&
           make_map(&mp.down, L.w_down, H, c.mlp, c.mlp, BM);
      if (ok && c.layer_is_attn[l])
        ok = make_map(&mp.q, L.w_q, qd, H, H, BM) && make_map(&mp.k, L.w_k, kd, H, H, BM) &&
             make_map(&mp.v, L.w_v, kd, H, H, BM) && make_map(&mp.out, L.w_o, H, qd, qd, BM);
      else if (ok)
        ok = make_map(&mp.in_proj, L.in_proj, m.rin, H, H, BM) &&
             make_map(&mp.out, L.out_proj, H, vd, vd, BM);
    }
    e->pf_ok = ok && (c.dn_dk == 64 || c.dn_dk == 128) && c.dn_dk == c.dn_dv &&
               (c.head_dim == 64 || c.head_dim == 128 || c.head_dim == 256);
  }
  int rc = mk_reset(e);
  if (rc != MK_OK) {
    delete e;
    return rc;
  }
  *out = e;
  return MK_OK;
}

void mk_destroy(mk_engine* e) { delete e; }

int mk_reset(mk_engine* e) {
  if (!e) return MK_ERR_ARG;
  const Layout& L = e->lay;
  cudaError_t r = cudaSuccess;
  // everything after the model struct up to (not including) the KV cache,
  // then activations and control words
  for (int b = 0; b < mk::kStateBufs && r == cudaSuccess; ++b) {
    r = cudaMemsetAsync(e->ws + L.dn_state[b], 0, L.conv_state[b] - L.dn_state[b], e->stream);
    if (r == cudaSuccess)
      r = cudaMemsetAsync(e->ws + L.conv_state[b], 0,
                          (b + 1 < mk::kStateBufs ? L.dn_state[b + 1] : L.kc) - L.conv_state[b],
                          e->stream);
  }
  if (r == cudaSuccess) r = cudaMemsetAsync(e->ws + L.xacc, 0, L.total - L.xacc, e->stream);
  if (r != cudaSuccess) return cuda_status(r);
  e->pos = 0;
  e->cur_buf = 0;
  e->amax_toggle = 0;
  e->amax_valid = false;
  e->pending_verify = 0;
  e->replay_n = 0;
  return MK_OK;
}

int mk_position(const mk_engine* e) { return e ? e->pos : -1; }

int mk_sync(mk_engine* e) {
  if (!e) return MK_ERR_ARG;
  cudaError_t r = cudaStreamSynchronize(e->stream);
  if (r != cudaSuccess) return cuda_status(r);
  int err = read_device_error(e);
  return err;
}

int mk_decode_step(mk_engine* e, int32_t token, float* logits_out) {
  if (!e) return MK_ERR_ARG;
  if (token < 0 || token >= e->cfg.vocab) return MK_ERR_ARG;
  if (e->pending_verify) return MK_ERR_STATE;
  if (e->pos + 1 > e->cfg.max_ctx) return MK_ERR_CTX_OVERFLOW;
  return decode_advance(e, token, 0, logits_out, nullptr);
}

int mk_generate(mk_engine* e, int32_t first_token, int n, int32_t* tokens_out,
                float* logits_out) {
  if (!e || n < 0 || !tokens_out) return MK_ERR_ARG;
  if (first_token < -1 || first_token >= e->cfg.vocab) return MK_ERR_ARG;
  if (first_token == -1 && !e->amax_valid) return MK_ERR_STATE;
  if (e->pending_verify) return MK_ERR_STATE;
  if (e->pos + n > e->cfg.max_ctx) return MK_ERR_CTX_OVERFLOW;
  for (int i = 0; i < n; ++i) {
    float* lg = logits_out ? logits_out + size_t(i) * e->cfg.vocab : nullptr;
    const int from_device = (i > 0 || first_token == -1) ? 1 : 0;
    int rc = decode_advance(e, first_token < 0 ? 0 : first_token, from_device, lg, tokens_out + i);
    if (rc != MK_OK) return rc;
  }
  return MK_OK;
}

int mk_prefill(mk_engine* e, const int32_t* tokens_host, int n, float* logits_out) {
  if (!e || n < 0 || (n > 0 && !tokens_host)) return MK_ERR_ARG;
  if (e->pending_verify) return MK_ERR_STATE;
  if (e->pos + n > e->cfg.max_ctx) return MK_ERR_CTX_OVERFLOW;
  for (int i = 0; i < n; ++i)
    if (tokens_host[i] < 0 || tokens_host[i] >= e->cfg.vocab) return MK_ERR_ARG;
  int i = 0;
  // all but the last position through the tensor-core path, in chunks
  if (e->pf_ok && n - 1 >= kPrefillMinBatch) {
    while (i < n - 1) {
      const int T = (n - 1 - i) < e->lay.tmax ? (n - 1 - i) : e->lay.tmax;
      const int rc = run_chunk(e, tokens_host + i, T, nullptr, nullptr);
      if (rc != MK_OK) return rc;
      i += T;
    }
  }
  // the rest (at least the last position: its logits and greedy argmax)
  for (; i < n; ++i) {
    int rc = decode_advance(e, tokens_host[i], 0, i == n - 1 ? logits_out : nullptr, nullptr);
    if (rc != MK_OK) return rc;
  }
  return MK_OK;
}

int mk_verify(mk_engine* e, const int32_t* tokens_host, int n, float* logits_out) {
  if (!e || !tokens_host || !logits_out || n < 1 || n > e->cfg.max_verify) return MK_ERR_ARG;
  if (e->pending_verify) return MK_ERR_STATE;
  if (e->pos + n > e->cfg.max_ctx) return MK_ERR_CTX_OVERFLOW;
  for (int i = 0; i < n; ++i)
    if (tokens_host[i] < 0 || tokens_host[i] >= e->cfg.vocab) return MK_ERR_ARG;
  if (e->pf_ok) {
    // one chunk: every projection one pass over its weights for the n
    // positions; the DeltaNet layers first replay what the last accept
    // kept, then record the chunk's positions for the next accept
    VerifyPlan vp;
    vp.R = e->replay_n;
    vp.rsel = e->replay_sel;
    vp.wsel = e->replay_sel ^ 1;
    vp.nb = vp.R > 0 ? (e->cur_buf + 1) % mk::kStateBufs : e->cur_buf;
    const int rc = run_chunk(e, tokens_host, n, &vp, logits_out);
    if (rc != MK_OK) return rc;
    e->cur_buf = vp.nb;
    e->replay_n = 0;
    e->vlog_sel = vp.wsel;
    e->verify_logged = true;
    e->pending_verify = n;
    e->amax_valid = false;
    return MK_OK;
  }
  e->verify_logged = false;
  // no chunk path: one decode launch per position, each reading the state
  // after the previous position and writing its own checkpoint buffer
  int src = e->cur_buf, k = 0;
  for (int j = 0; j < n; ++j) {
    const int dst = (e->cur_buf + 1 + j) % mk::kStateBufs;
    e->verify_bufs[j] = dst;
    int rc = launch_decode(e, e->pos + j, src, dst, tokens_host[j], 0,
                           logits_out + size_t(j) * e->cfg.vocab, nullptr);
    if (rc != MK_OK) return rc;
    src = dst;
    ++k;
  }
  e->pending_verify = k;
  e->amax_valid = false;  // the argmax is position n-1's; accept may keep fewer
  return MK_OK;
}

int mk_accept(mk_engine* e, int n_keep) {
  if (!e) return MK_ERR_ARG;
  if (!e->pending_verify) return MK_ERR_STATE;
  if (n_keep < 1 || n_keep > e->pending_verify) return MK_ERR_ARG;
  if (e->verify_logged) {
    e->replay_n = n_keep;  // applied by the next call that reads the state
    e->replay_sel = e->vlog_sel;
  } else {
    e->cur_buf = e->verify_bufs[n_keep - 1];
  }
  e->pos += n_keep;
  e->pending_verify = 0;
  return MK_OK;
}

int32_t mk_last_argmax(mk_engine* e) {
  if (!e || e->launches == 0) return -1;
  unsigned long long v = 0;
  if (cudaStreamSynchronize(e->stream) != cudaSuccess ||
      cudaMemcpy(&v, e->ws + e->lay.amax + 8 * e->amax_toggle, 8, cudaMemcpyDeviceToHost) !=
          cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  if (!v) return -1;
  return int32_t(0xFFFFFFFFu - uint32_t(v & 0xFFFFFFFFull));
}

int mk_set_state(mk_engine* e, int pos, const float* dn_state, const float* conv_state,
                 const void* k_cache, const void* v_cache) {
  if (!e || pos < 0 || pos > e->cfg.max_ctx || !dn_state || !conv_state) return MK_ERR_ARG;
  if (pos > 0 && (!k_cache || !v_cache)) return MK_ERR_ARG;
  int rc = mk_reset(e);
  if (rc != MK_OK) return rc;
  const Layout& L = e->lay;
  const DevModel& m = e->hm;
  const size_t dn_bytes = size_t(m.n_dn) * m.nh * m.dv * m.dk * 4;
  cudaError_t r = cudaMemcpyAsync(e->ws + L.dn_state[0], dn_state, dn_bytes,
                                  cudaMemcpyDeviceToDevice, e->stream);
  const size_t rows = size_t(m.n_dn) * m.ch;
  if (r == cudaSuccess && rows)
    r = cudaMemcpy2DAsync(e->ws + L.conv_state[0], 16, conv_state, 12, 12, rows,
                          cudaMemcpyDeviceToDevice, e->stream);
  const size_t heads = size_t(m.n_attn) * m.nkv;
  if (r == cudaSuccess && pos > 0 && heads) {
    const size_t w = size_t(pos) * m.hd * 2, dp = size_t(m.max_ctx) * m.hd * 2;
    r = cudaMemcpy2DAsync(e->ws + L.kc, dp, k_cache, w, w, heads, cudaMemcpyDeviceToDevice,
                          e->stream);
    if (r == cudaSuccess)
      r = cudaMemcpy2DAsync(e->ws + L.vc, dp, v_cache, w, w, heads, cudaMemcpyDeviceToDevice,
                            e->stream);
  }
  if (r != cudaSuccess) return cuda_status(r);
  e->pos = pos;
  return MK_OK;
}

int mk_get_state(mk_engine* e, float* dn_state, float* conv_state, void* k_cache,
                 void* v_cache) {
  if (!e) return MK_ERR_ARG;
  const int rp = replay_pending(e);
  if (rp != MK_OK) return rp;
  const Layout& L = e->lay;
  const DevModel& m = e->hm;
  const int b = e->cur_buf;
  cudaError_t r = cudaSuccess;
  if (dn_state)
    r = cudaMemcpyAsync(dn_state, e->ws + L.dn_state[b], size_t(m.n_dn) * m.nh * m.dv * m.dk * 4,
                        cudaMemcpyDeviceToDevice, e->stream);
  const size_t rows = size_t(m.n_dn) * m.ch;
  if (r == cudaSuccess && conv_state && rows)
    r = cudaMemcpy2DAsync(conv_state, 12, e->ws + L.conv_state[b], 16, 12, rows,
                          cudaMemcpyDeviceToDevice, e->stream);
  const size_t heads = size_t(m.n_attn) * m.nkv;
  if (r == cudaSuccess && e->pos > 0 && heads) {
    const size_t w = size_t(e->pos) * m.hd * 2, sp = size_t(m.max_ctx) * m.hd * 2;
    if (k_cache)
      r = cudaMemcpy2DAsync(k_cache, w, e->ws + L.kc, sp, w, heads, cudaMemcpyDeviceToDevice,
                            e->stream);
    if (r == cudaSuccess && v_cache)
      r = cudaMemcpy2DAsync(v_cache, w, e->ws + L.vc, sp, w, heads, cudaMemcpyDeviceToDevice,
                            e->stream);
  }
  return cuda_status(r);
}

int mk_get_hidden(mk_engine* e, float* hidden_out) {
  if (!e || !hidden_out) return MK_ERR_ARG;
  return cuda_status(cudaMemcpyAsync(hidden_out, e->ws + e->lay.hidden,
                                     size_t(e->cfg.n_layers) * e->cfg.hidden * 4,
                                     cudaMemcpyDeviceToDevice, e->stream));
}

int64_t mk_launch_count(const mk_engine* e) { return e ? e->launches : -1; }

int mk_debug_set_wait_limit(mk_engine* e, int64_t limit_ns, int fail_phase) {
  if (!e || limit_ns <= 0) return MK_ERR_ARG;
  e->wait_ns = limit_ns;
  e->fail_phase = fail_phase;
  return MK_OK;
}

int mk_delta_step(float* S, const void* q, const void* k, const void* v, const float* alpha,
                  const float* beta, float* o, int B, int heads, int dk, int dv, void* stream) {
  if (!S || !q || !k || !v || !alpha || !beta || !o || B <= 0 || heads <= 0) return MK_ERR_ARG;
  if (dk != dv || (dk != 64 && dk != 128)) return MK_ERR_UNSUPPORTED;
  if (!aligned16(S)) return MK_ERR_ARG;
  dim3 grid(unsigned(B) * unsigned(heads), unsigned(dv / mk::DS_ROWS));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint16_t* q16 = static_cast<const uint16_t*>(q);
  const uint16_t* k16 = static_cast<const uint16_t*>(k);
  const uint16_t* v16 = static_cast<const uint16_t*>(v);
  if (dk == 128)
    mk::delta_step_kernel<128><<<grid, mk::DS_THREADS, 0, st>>>(S, q16, k16, v16, alpha, beta, o);
  else
    mk::delta_step_kernel<64><<<grid, mk::DS_THREADS, 0, st>>>(S, q16, k16, v16, alpha, beta, o);
  return cuda_status(cudaGetLastError());
}

size_t mk_delta_chunked_ws_bytes(int T, int heads, int dk) {
  if (T <= 0 || heads <= 0 || (dk != 64 && dk != 128)) return 0;
  const size_t nc = (size_t(T) + mk::ck::C - 1) / mk::ck::C;
  const size_t blk = dk == 64 ? mk::ck::Blk<64>::FLOATS : mk::ck::Blk<128>::FLOATS;
  return align256(size_t(heads) * T * 2 * dk * 4) + align256(size_t(heads) * T * 16) +
         size_t(heads) * nc * blk * 4;
}

int mk_delta_chunked(float* S, const float* q, const float* k, const float* v,
                     const float* alpha, const float* beta, float* o, int T, int heads, int dk,
                     int dv, void* workspace, size_t ws_bytes, void* stream) {
  if (!S || !q || !k || !v || !alpha || !beta || !o || !workspace || T <= 0 || heads <= 0)
    return MK_ERR_ARG;
  if (dk != dv || (dk != 64 && dk != 128)) return MK_ERR_UNSUPPORTED;
  if (!aligned16(S) || !aligned16(workspace) || ws_bytes < mk_delta_chunked_ws_bytes(T, heads, dk))
    return MK_ERR_ARG;
  static bool attr_done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  if (!attr_done[dev]) {
    if (cudaFuncSetAttribute(mk::ck::chunk_prep_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(mk::ck::prep_smem<128>())) != cudaSuccess ||
        cudaFuncSetAttribute(mk::ck::chunk_scan_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(mk::ck::scan_smem<128>())) != cudaSuccess ||
        cudaFuncSetAttribute(mk::ck::chunk_prep_kernel<64>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(mk::ck::prep_smem<64>())) != cudaSuccess ||
        cudaFuncSetAttribute(mk::ck::chunk_scan_kernel<64>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(mk::ck::scan_smem<64>())) != cudaSuccess) {
      cudaGetLastError();
      return MK_ERR_CUDA;
    }
    attr_done[dev] = true;
  }
  char* ws = static_cast<char*>(workspace);
  float* QK = reinterpret_cast<float*>(ws);
  float4* BAK = reinterpret_cast<float4*>(ws + align256(size_t(heads) * T * 2 * dk * 4));
  float* prep = reinterpret_cast<float*>(ws + align256(size_t(heads) * T * 2 * dk * 4) +
                                         align256(size_t(heads) * T * 16));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n_pos = size_t(heads) * T;
  const int pb = int((n_pos * dk + 255) / 256 < 4096 ? (n_pos * dk + 255) / 256 : 4096);
  const dim3 pg((T + mk::ck::C - 1) / mk::ck::C, heads), sg(dv / mk::ck::SCAN_ROWS, heads);
  // v and o are [heads][T][dv]: position stride dv, head stride T * dv
  const size_t ts = size_t(dv), hs = size_t(T) * dv;
  if (dk == 128) {
    mk::ck::chunk_pack_kernel<128><<<pb, 256, 0, st>>>(q, k, alpha, beta, n_pos, QK, BAK);
    mk::ck::chunk_prep_kernel<128><<<pg, mk::ck::PREP_THREADS, mk::ck::prep_smem<128>(), st>>>(
        QK, BAK, v, ts, hs, T, prep);
    mk::ck::chunk_scan_kernel<128><<<sg, mk::ck::SCAN_THREADS, mk::ck::scan_smem<128>(), st>>>(
        S, prep, T, o, ts, hs);
  } else {
    mk::ck::chunk_pack_kernel<64><<<pb, 256, 0, st>>>(q, k, alpha, beta, n_pos, QK, BAK);
    mk::ck::chunk_prep_kernel<64><<<pg, mk::ck::PREP_THREADS, mk::ck::prep_smem<64>(), st>>>(
        QK, BAK, v, ts, hs, T, prep);
    mk::ck::chunk_scan_kernel<64><<<sg, mk::ck::SCAN_THREADS, mk::ck::scan_smem<64>(), st>>>(
        S, prep, T, o, ts, hs);
  }
  return cuda_status(cudaGetLastError());
}

int mk_debug_gemm(const void* W, const void* X, float* C, int n_out, int T, int K,
                  void* stream) {
  if (!W || !X || !C || n_out <= 0 || T <= 0 || K <= 0 || K % 64) return MK_ERR_ARG;
  mk::pf::GemmArgs g;
  if (!make_map(&g.tw, W, n_out, K, K, mk::pf::BM) ||
      !make_map(&g.tx, X, 2 * T, K, K, mk::pf::BN))
    return MK_ERR_UNSUPPORTED;
  // a 4-byte wait-error word per device, allocated by the first call there
  static int* err_words[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  if (!err_words[dev] && cudaMalloc(&err_words[dev], 4) != cudaSuccess) return MK_ERR_CUDA;
  int* err_word = err_words[dev];
  if (cudaFuncSetAttribute(mk::pf::gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(mk::pf::GEMM_SMEM)) != cudaSuccess)
    return MK_ERR_CUDA;
  g.c = C;
  g.ldc = n_out;
  g.n_out = n_out;
  g.T = T;
  g.K = K;
  g.accumulate = 0;
  g.x_lo_row = T;
  g.k_split = 1;
  g.err = err_word;
  g.wait_ns = 2000000000LL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the error word starts each call at zero (stream-ordered); a tile that
  // gives up sets it and C is then filled with NaN
  const cudaError_t mr = cudaMemsetAsync(err_word, 0, 4, st);
  if (mr != cudaSuccess) return cuda_status(mr);
  const dim3 grid((n_out + mk::pf::BM - 1) / mk::pf::BM, (T + mk::pf::BN - 1) / mk::pf::BN);
  mk::pf::gemm_tc<<<grid, mk::pf::GEMM_THREADS, mk::pf::GEMM_SMEM, st>>>(g);
  const size_t n = size_t(T) * n_out;
  mk::pf::poison_on_error_kernel<<<int((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024), 256, 0,
                                   st>>>(err_word, n, C);
  return cuda_status(cudaGetLastError());
}

}  // extern "C"

namespace {
// Static device scratch of the allocation-free GEMM entry point: split-K
// partial sums (at most kNoAllocFloats floats = 8 MiB) and its wait-error
// word (cleared at the start of every call; set when a wait runs out).
constexpr size_t kNoAllocFloats = size_t(2) << 20;
__device__ __align__(256) float g_noalloc_partial[kNoAllocFloats];
__device__ __align__(256) int g_noalloc_err;
constexpr int kNoAllocMaxDevices = 64;
float* g_partial_addr[kNoAllocMaxDevices];
int* g_err_addr[kNoAllocMaxDevices];
}  // namespace

extern "C" {

int mk_debug_gemm_noalloc(const void* W, const void* X, float* C, int n_out, int T, int K,
                          void* stream) {
  if (!W || !X || !C || n_out <= 0 || T <= 0 || K <= 0 || K % 64) return MK_ERR_ARG;
  if (size_t(T) * size_t(n_out) > kNoAllocFloats) return MK_ERR_ARG;  // exceeds the static scratch
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  if (!g_partial_addr[dev]) {
    // first call on this device (the device is current): look up the scratch
    void* pp = nullptr;
    void* pe = nullptr;
    if (cudaGetSymbolAddress(&pp, g_noalloc_partial) != cudaSuccess ||
        cudaGetSymbolAddress(&pe, g_noalloc_err) != cudaSuccess) {
      cudaGetLastError();
      return MK_ERR_CUDA;
    }
    g_err_addr[dev] = static_cast<int*>(pe);
    g_partial_addr[dev] = static_cast<float*>(pp);
  }
  mk::pf::GemmArgs g;
  if (!make_map(&g.tw, W, n_out, K, K, mk::pf::BM) ||
      !make_map(&g.tx, X, 2 * T, K, K, mk::pf::BN))
    return MK_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(mk::pf::gemm_tc_partial, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(mk::pf::GEMM_SMEM)) != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  int sms = 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms = 148;
  const int tiles = ((n_out + mk::pf::BM - 1) / mk::pf::BM) * ((T + mk::pf::BN - 1) / mk::pf::BN);
  int ks = (sms + tiles - 1) / tiles;
  if (ks > K / mk::pf::BK) ks = K / mk::pf::BK;
  while (ks > 1 && size_t(ks) * T * n_out > kNoAllocFloats) --ks;
  if (ks < 1) ks = 1;
  g.c = C;
  g.ldc = n_out;
  g.n_out = n_out;
  g.T = T;
  g.K = K;
  g.accumulate = 0;
  g.x_lo_row = T;
  g.k_split = ks;
  g.err = g_err_addr[dev];
  g.wait_ns = 2000000000LL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the error word starts each call at zero (stream-ordered, no allocation);
  // a range that gives up sets it and the reduction then writes NaN
  const cudaError_t mr = cudaMemsetAsync(g_err_addr[dev], 0, 4, st);
  if (mr != cudaSuccess) return cuda_status(mr);
  const dim3 grid((n_out + mk::pf::BM - 1) / mk::pf::BM, (T + mk::pf::BN - 1) / mk::pf::BN, ks);
  mk::pf::gemm_tc_partial<<<grid, mk::pf::GEMM_THREADS, mk::pf::GEMM_SMEM, st>>>(
      g, g_partial_addr[dev]);
  const size_t n = size_t(T) * n_out;
  const int rblocks = int((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  mk::pf::splitk_reduce_kernel<<<rblocks, 256, 0, st>>>(g_partial_addr[dev], ks, n, C,
                                                        g_err_addr[dev]);
  return cuda_status(cudaGetLastError());
}

int mk_quantize_w4(const void* W, int rows, int cols, void* codes, float* scales, void* stream) {
  if (!W || !codes || !scales || rows <= 0 || cols <= 0 || cols % mk::q4::G) return MK_ERR_ARG;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(scales)) return MK_ERR_ARG;
  const size_t groups = size_t(rows) * (cols / mk::q4::G);
  const size_t blocks = (groups + 255) / 256;
  if (blocks > 0x7FFFFFFFu) return MK_ERR_UNSUPPORTED;
  mk::q4::quantize_w4_kernel<<<unsigned(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(W), rows, cols, static_cast<uint8_t*>(codes), scales);
  return cuda_status(cudaGetLastError());
}

int mk_gemv_w4(const void* codes, const float* scales, const float* x, int T, int rows, int cols,
               float* y, void* stream) {
  if (!codes || !scales || !x || !y || T < 1 || T > mk::q4::TMAX || rows <= 0 || cols <= 0 ||
      cols % mk::q4::G)
    return MK_ERR_ARG;
  if (!aligned16(codes) || !aligned16(x) || (reinterpret_cast<uintptr_t>(scales) & 3u) ||
      (reinterpret_cast<uintptr_t>(y) & 3u))
    return MK_ERR_ARG;
  const size_t smem = size_t(T) * cols * 4;  // the T activation rows
  if (smem > 220u * 1024u) return MK_ERR_UNSUPPORTED;
  int dev = 0;
  cudaError_t r = cudaGetDevice(&dev);
  if (r != cudaSuccess) return cuda_status(r);
  // the dynamic shared memory limit, raised per device and token count when a
  // call needs more than the last one did
  static size_t attr_smem[64][mk::q4::TMAX + 1] = {};
  if (dev < 0 || dev >= 64) return MK_ERR_UNSUPPORTED;
  if (attr_smem[dev][T] < smem) {
    const void* fns[mk::q4::TMAX + 1] = {
        nullptr,
        reinterpret_cast<const void*>(mk::q4::gemv_w4_kernel<1>),
        reinterpret_cast<const void*>(mk::q4::gemv_w4_kernel<2>),
        reinterpret_cast<const void*>(mk::q4::gemv_w4_kernel<3>),
        reinterpret_cast<const void*>(mk::q4::gemv_w4_kernel<4>),
        reinterpret_cast<const void*>(mk::q4::gemv_w4_kernel<5>),
        reinterpret_cast<const void*>(mk::q4::gemv_w4_kernel<6>),
        reinterpret_cast<const void*>(mk::q4::gemv_w4_kernel<7>),
        reinterpret_cast<const void*>(mk::q4::gemv_w4_kernel<8>)};
    r = cudaFuncSetAttribute(fns[T], cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (r != cudaSuccess) return cuda_status(r);
    attr_smem[dev][T] = smem;
  }
  const int kw = mk::q4::pick_kw(cols);
  const int rw = mk::q4::rw_for(T);
  const int rpb = (mk::q4::WARPS / kw) * rw;
  const int nblk = (rows + rpb - 1) / rpb;
  const dim3 grid(nblk < mk::q4::MAX_CTAS ? nblk : mk::q4::MAX_CTAS), block(mk::q4::THREADS);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint8_t* c = static_cast<const uint8_t*>(codes);
  switch (T) {
    case 1: mk::q4::gemv_w4_kernel<1><<<grid, block, smem, st>>>(c, scales, x, rows, cols, y, kw); break;
    case 2: mk::q4::gemv_w4_kernel<2><<<grid, block, smem, st>>>(c, scales, x, rows, cols, y, kw); break;
    case 3: mk::q4::gemv_w4_kernel<3><<<grid, block, smem, st>>>(c, scales, x, rows, cols, y, kw); break;
    case 4: mk::q4::gemv_w4_kernel<4><<<grid, block, smem, st>>>(c, scales, x, rows, cols, y, kw); break;
    case 5: mk::q4::gemv_w4_kernel<5><<<grid, block, smem, st>>>(c, scales, x, rows, cols, y, kw); break;
    case 6: mk::q4::gemv_w4_kernel<6><<<grid, block, smem, st>>>(c, scales, x, rows, cols, y, kw); break;
    case 7: mk::q4::gemv_w4_kernel<7><<<grid, block, smem, st>>>(c, scales, x, rows, cols, y, kw); break;
    default: mk::q4::gemv_w4_kernel<8><<<grid, block, smem, st>>>(c, scales, x, rows, cols, y, kw); break;
  }
  return cuda_status(cudaGetLastError());
}

const char* mk_strerror(int s) {
  switch (s) {
    case MK_OK: return "ok";
    case MK_ERR_ARG: return "invalid argument";
    case MK_ERR_CTX_OVERFLOW: return "KV cache capacity exceeded";
    case MK_ERR_STATE: return "call not valid in the engine's current state";
    case MK_ERR_LAUNCH: return "cooperative launch impossible or failed";
    case MK_ERR_TIMEOUT: return "device-side wait gave up";
    case MK_ERR_CUDA: return "CUDA runtime error";
    case MK_ERR_UNSUPPORTED: return "shape not implemented by the kernels";
    case MK_ERR_RANGE: return "decode partial sum outside the fixed-point range";
    default: return "unknown status";
  }
}

}  // extern "C"
