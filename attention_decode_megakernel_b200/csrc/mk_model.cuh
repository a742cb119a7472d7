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
  const uint16_t *mlp_norm, *w_gate, *w_up, *w_down;
  // engine copies laid out for the decode kernel's group partition
  const uint16_t* w_qkv;       // attention q|k|v rows, [(nq + 2 nkv) hd][H]
  const uint16_t* w_in_pk;     // DeltaNet in-proj rows per head, [nh][q|k|v|z|b|a][H]
  const uint16_t* w_out_blk;   // output projection by K block, [ng][H][K / ng]
  const uint16_t* w_down_blk;  // MLP down projection by K block, [ng][H][I / ng]
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
  int ng, gs;                       // decode groups (one per DeltaNet head) and CTAs per group
  int rin_h, kb_att, kb_mlp;        // in-proj rows per head; K block of the attention / MLP partials
  float eps, theta;
  // weights
  const uint16_t *embed, *final_norm;
  DevLayer layers[MK_MAX_LAYERS];
  // recurrent state: kStateBufs rotating buffers (current, next, and the
  // per-position copies of the decode-launch verify fallback)
  float *dn_state[kStateBufs];      // [n_dn][nh][dv][dk]
  float *conv_state[kStateBufs];    // [n_dn][ch][4]  (3 taps of history + pad)
  uint16_t *kc, *vc;                // [n_attn][nkv][max_ctx][hd]
  // decode exchange buffers: tagged words {fp32 value, tag} and count-carrying
  // fixed-point sums (see mk_decode.cuh)
  unsigned long long *xacc;     // [2 launch parities][n_layers][2][H] residual deltas
  unsigned long long *grp_inp;  // [ng][rin_h] one head's in-projection outputs
  unsigned long long *grp_h;    // [ng][I / ng] one group's SiLU(gate)*up values
  unsigned long long *qkv_ll;   // [(nq+2nkv)*hd] raw attention projections
  unsigned long long *part_ll;  // [nkv][kMaxCtas][group][hd+2] split-K attention partials
  float *hidden;   // [n_layers][H] residual after each layer (last position)
  float *logits_scratch;  // [V]
  unsigned *tickets;      // [1] grid argmax ticket
  int *err;               // first device error code
  unsigned long long *amax;  // [2] packed argmax slots
};

}  // namespace mk
