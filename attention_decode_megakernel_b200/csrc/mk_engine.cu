// mk_engine.cu -- host side of the C ABI declared in include/mk.h: config
// validation, workspace carve-up, cooperative launches of the decode kernel,
// state rotation for verify checkpoints, state I/O and error reporting.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <new>

#include "mk.h"
#include "mk_decode.cuh"
#include "mk_delta.cuh"
#include "mk_model.cuh"

namespace {

using mk::DevModel;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Layout {
  size_t model;
  size_t dn_state[mk::kStateBufs], conv_state[mk::kStateBufs];
  size_t kc, vc;
  size_t x, inp, dno, qkv, atto, mlph, part, hidden, logits, tickets, err, amax;
  size_t total;
};

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
  const size_t M = size_t(c.max_verify);
  const size_t G = size_t(c.q_heads / c.kv_heads);
  L.model = take(sizeof(DevModel));
  for (int b = 0; b < mk::kStateBufs; ++b) {
    L.dn_state[b] = take(size_t(n_dn) * c.dn_heads * c.dn_dv * c.dn_dk * 4);
    L.conv_state[b] = take(size_t(n_dn) * ch * 4 * 4);
  }
  const size_t kv = size_t(n_attn) * c.kv_heads * c.max_ctx * c.head_dim * 2;
  L.kc = take(kv);
  L.vc = take(kv);
  L.x = take(2 * M * c.hidden * 8);
  L.inp = take(M * rin * 8);
  L.dno = take(M * c.dn_heads * c.dn_dv * 8);
  L.qkv = take(M * size_t(c.q_heads + 2 * c.kv_heads) * c.head_dim * 8);
  L.atto = take(M * size_t(c.q_heads) * c.head_dim * 8);
  L.mlph = take(M * size_t(c.mlp) * 8);
  L.part = take(size_t(c.kv_heads) * mk::kMaxCtas * M * G * (c.head_dim + 2) * 8);
  L.hidden = take(size_t(c.n_layers) * c.hidden * 4);
  L.logits = take(size_t(c.vocab) * 4);
  L.tickets = take(4);
  L.err = take(4);
  L.amax = take(2 * 8);
  L.total = off;
  return L;
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
  int pending_verify;
  int verify_bufs[mk::kMaxVerify];
  int64_t launches;
  long long wait_ns;
  int fail_phase;
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

int launch_decode(mk_engine* e, int pos, int st_buf, int token, int tok_src, float* logits,
                  int32_t* tok_out) {
  mk::StepArgs a;
  a.m = e->hm;
  a.pos = pos;
  a.token = token;
  a.tok_src = tok_src;
  a.amax_in = e->amax_toggle;
  a.amax_out = e->amax_toggle ^ 1;
  a.st_buf = st_buf;
  a.logits = logits ? logits : reinterpret_cast<float*>(e->ws + e->lay.logits);
  a.tok_out = tok_out;
  a.hidden = reinterpret_cast<float*>(e->ws + e->lay.hidden);
  e->seq = e->seq + 1 >= (1u << 23) ? 1u : e->seq + 1;
  a.seq = e->seq;
  a.fail_phase = e->fail_phase;
  a.wait_ns = e->wait_ns;
  e->fail_phase = -1;
  void* args[] = {&a};
  cudaError_t err = cudaLaunchCooperativeKernel(e->var->fn, dim3(e->ncta), dim3(mk::NTHR), args,
                                                e->var->smem, e->stream);
  if (err != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_LAUNCH;
  }
  e->amax_toggle ^= 1;
  e->launches += 1;
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
  {
    // attention merge scratch: (m, l) and weights of every split
    const int smax = ncta / c.kv_heads;
    const int att = 2 * G * c.head_dim + 2 * c.head_dim + mk::NCW * G * 2;
    if (att + smax * G * 3 > mk::UNION_FLOATS || G * c.head_dim + smax > att)
      return MK_ERR_UNSUPPORTED;
  }
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
  // the DeltaNet head cache, row values and conv staging must fit a CTA's
  // shared scratch
  if ((2 * c.dn_heads * c.dn_dk + 2 * c.dn_heads * c.dn_dv + 2 * c.dn_heads + ncta - 1) / ncta >
      mk::CONV_ROWS_MAX)
    return MK_ERR_UNSUPPORTED;
  {
    int rows = (c.dn_heads * c.dn_dv + ncta - 1) / ncta;
    int heads = rows / c.dn_dv + 2;
    if (heads > mk::DN_HEADS_MAX || rows > mk::DN_ROWS_MAX) return MK_ERR_UNSUPPORTED;
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
  using ull = unsigned long long;
  m.x_ll = reinterpret_cast<ull*>(ws + lay.x);
  m.inp_ll = reinterpret_cast<ull*>(ws + lay.inp);
  m.dno_ll = reinterpret_cast<ull*>(ws + lay.dno);
  m.qkv_ll = reinterpret_cast<ull*>(ws + lay.qkv);
  m.atto_ll = reinterpret_cast<ull*>(ws + lay.atto);
  m.mlph_ll = reinterpret_cast<ull*>(ws + lay.mlph);
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
  if (r == cudaSuccess) r = cudaMemsetAsync(e->ws + L.x, 0, L.total - L.x, e->stream);
  if (r != cudaSuccess) return cuda_status(r);
  e->pos = 0;
  e->cur_buf = 0;
  e->amax_toggle = 0;
  e->pending_verify = 0;
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
  int rc = launch_decode(e, e->pos, e->cur_buf, token, 0, logits_out, nullptr);
  if (rc == MK_OK) e->pos += 1;
  return rc;
}

int mk_generate(mk_engine* e, int32_t first_token, int n, int32_t* tokens_out,
                float* logits_out) {
  if (!e || n < 0 || !tokens_out) return MK_ERR_ARG;
  if (first_token < -1 || first_token >= e->cfg.vocab) return MK_ERR_ARG;
  if (first_token == -1 && e->launches == 0) return MK_ERR_STATE;
  if (e->pending_verify) return MK_ERR_STATE;
  if (e->pos + n > e->cfg.max_ctx) return MK_ERR_CTX_OVERFLOW;
  for (int i = 0; i < n; ++i) {
    float* lg = logits_out ? logits_out + size_t(i) * e->cfg.vocab : nullptr;
    const int from_device = (i > 0 || first_token == -1) ? 1 : 0;
    int rc = launch_decode(e, e->pos, e->cur_buf, first_token < 0 ? 0 : first_token, from_device,
                           lg, tokens_out + i);
    if (rc != MK_OK) return rc;
    e->pos += 1;
  }
  return MK_OK;
}

int mk_prefill(mk_engine* e, const int32_t* tokens_host, int n, float* logits_out) {
  if (!e || n < 0 || (n > 0 && !tokens_host)) return MK_ERR_ARG;
  if (e->pending_verify) return MK_ERR_STATE;
  if (e->pos + n > e->cfg.max_ctx) return MK_ERR_CTX_OVERFLOW;
  for (int i = 0; i < n; ++i)
    if (tokens_host[i] < 0 || tokens_host[i] >= e->cfg.vocab) return MK_ERR_ARG;
  for (int i = 0; i < n; ++i) {
    int rc = launch_decode(e, e->pos, e->cur_buf, tokens_host[i], 0,
                           i == n - 1 ? logits_out : nullptr, nullptr);
    if (rc != MK_OK) return rc;
    e->pos += 1;
  }
  return MK_OK;
}

int mk_verify(mk_engine* e, const int32_t* tokens_host, int n, float* logits_out) {
  if (!e || !tokens_host || !logits_out || n < 1 || n > e->cfg.max_verify) return MK_ERR_ARG;
  if (e->pending_verify) return MK_ERR_STATE;
  if (e->pos + n > e->cfg.max_ctx) return MK_ERR_CTX_OVERFLOW;
  for (int i = 0; i < n; ++i)
    if (tokens_host[i] < 0 || tokens_host[i] >= e->cfg.vocab) return MK_ERR_ARG;
  const Layout& L = e->lay;
  const size_t dn_bytes = L.conv_state[0] - L.dn_state[0];
  const size_t conv_bytes = (mk::kStateBufs > 1 ? L.dn_state[1] : L.kc) - L.conv_state[0];
  int src = e->cur_buf, k = 0;
  for (int j = 0; j < n; ++j) {
    int dst = (e->cur_buf + 1 + j) % mk::kStateBufs;
    e->verify_bufs[j] = dst;
    cudaError_t r = cudaMemcpyAsync(e->ws + L.dn_state[dst], e->ws + L.dn_state[src], dn_bytes,
                                    cudaMemcpyDeviceToDevice, e->stream);
    if (r == cudaSuccess)
      r = cudaMemcpyAsync(e->ws + L.conv_state[dst], e->ws + L.conv_state[src], conv_bytes,
                          cudaMemcpyDeviceToDevice, e->stream);
    if (r != cudaSuccess) return cuda_status(r);
    int rc = launch_decode(e, e->pos + j, dst, tokens_host[j], 0,
                           logits_out + size_t(j) * e->cfg.vocab, nullptr);
    if (rc != MK_OK) return rc;
    src = dst;
    ++k;
  }
  e->pending_verify = k;
  return MK_OK;
}

int mk_accept(mk_engine* e, int n_keep) {
  if (!e) return MK_ERR_ARG;
  if (!e->pending_verify) return MK_ERR_STATE;
  if (n_keep < 1 || n_keep > e->pending_verify) return MK_ERR_ARG;
  e->cur_buf = e->verify_bufs[n_keep - 1];
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
    default: return "unknown status";
  }
}

}  // extern "C"
