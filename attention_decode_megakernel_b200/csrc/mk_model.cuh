// mk_model.cuh -- device-side description of one engine: shapes, weight
// pointers and the carve-up of the caller's workspace.  The struct lives in
// device memory (written once by mk_create); kernels receive a pointer.
#pragma once
#include <cstdint>

#include "mk.h"

namespace mk {

constexpr int kMaxVerify = 8;      // tokens per verify launch
constexpr int kStateBufs = kMaxVerify + 1;
constexpr int kMaxCtas = 256;      // upper bound of the persistent grid

struct DevLayer {
  const uint16_t *attn_norm, *in_proj, *conv_w;
  const float *A_log, *dt_bias;
  const uint16_t *out_norm, *out_proj;
  const uint16_t *w_q, *w_k, *w_v, *w_o;
  const uint16_t* w_qkv;  // engine copy of q|k|v rows, [(nq + 2 nkv) hd][H]
  const uint16_t *mlp_norm, *w_gate, *w_up, *w_down;
  int is_attn;
  int sub;  // index among layers of the same kind
};

struct DevModel {
  // shapes
  int n_layers, n_dn, n_attn;
  int H, V, I;
  int nh, dk, dv, ck, ch, rin;      // DeltaNet: heads, dims, conv taps/channels, in_proj rows
  int nq, nkv, hd;                  // attention
  int max_ctx, max_verify, ncta;
  float eps, theta;
  // weights
  const uint16_t *embed, *final_norm;
  DevLayer layers[MK_MAX_LAYERS];
  // recurrent state: kStateBufs rotating buffers (current + verify checkpoints)
  float *dn_state[kStateBufs];      // [n_dn][nh][dv][dk]
  float *conv_state[kStateBufs];    // [n_dn][ch][4]  (3 taps of history + pad)
  uint16_t *kc, *vc;                // [n_attn][nkv][max_ctx][hd]
  // activations exchanged between CTAs, as tagged words {fp32 value, tag}
  // (M = max_verify rows where noted)
  unsigned long long *x_ll;     // [2][M][H]  residual stream (double-buffered)
  unsigned long long *inp_ll;   // [M][rin]   in-proj output: conv'd q|k|v, raw z|b|a
  unsigned long long *dno_ll;   // [M][nh*dv] DeltaNet readout o = S q
  unsigned long long *qkv_ll;   // [M][(nq+2nkv)*hd] raw attention projections
  unsigned long long *atto_ll;  // [M][nq*hd] attention output (merged)
  unsigned long long *mlph_ll;  // [M][I]     SiLU(gate)*up
  unsigned long long *part_ll;  // [nkv][kMaxCtas][M*group][hd+2] split-K attention partials (tagged)
  float *hidden;   // [n_layers][H] residual after each layer (last position)
  float *logits_scratch;  // [V]
  unsigned *tickets;      // [1] grid argmax ticket
  int *err;               // first device error code
  unsigned long long *amax;  // [2] packed argmax slots
};

}  // namespace mk
