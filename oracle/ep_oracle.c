/*
 * CPU oracle for MoE expert-parallel dispatch / combine.
 *
 * TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg are the only callers.  Plain, slow, obviously
 * correct single-threaded C; shares nothing with the CUDA library.
 *
 * Sources (the pages describe the operations; they print no formula):
 *  - dispatch sends every token to the k experts its router chose; combine
 *    brings the k expert outputs back to the token's rank and sums them; the
 *    handle saved by dispatch is reused by combine and by the two backward
 *    passes: "DeepEP：MoE 专家并行 EP 通信 kernel 编译与使用指南"
 *    (zhouruolin.cn), section 五 使用方法 and FAQ Q5.
 *  - per-expert token counts as the load-skew diagnostic: "DeepEP：专为MoE模型
 *    打造的All-to-All通信库" (bjdmk.com.cn), section 5.2.
 *  - FP8 dispatch with BF16 combine as the standard precision pair:
 *    "deepep-expert-parallel-communication-library" (blog.hotdry.top),
 *    section 五 实践建议; "DeepSeek 开源周第二弹" (czhn.yksolo.com) (原生 FP8
 *    调度支持).
 *  - quantisation fused into the data movement: "DeepEP：专为MoE模型打造的
 *    All-to-All通信库", section 3.2.
 *
 * Readings where the pages are silent (each one is a choice, stated here):
 *  - FP8 is OCP E4M3 ("fn": bias 7, 3 mantissa bits, no infinity, S.1111.111
 *    is NaN, largest finite 448).  One fp32 scale per token per 128 channels:
 *    scale = amax / 448 (fp32 division); if that is 0, scale = 1.
 *    Code = E4M3(x / scale), fp32 division, round to nearest even, values
 *    beyond 448 saturate to 448 (sign kept; -0 encodes as 0x80).
 *  - Slots: the pairs routed to expert e occupy rows
 *    [expert_offset[e], expert_offset[e+1]) of the receive buffer, in
 *    increasing (token, top-k position) order.  Because virtual rank r owns
 *    the contiguous token range [r*T/R, (r+1)*T/R), this is also
 *    (source rank, source token) order.  Expert e belongs to rank e / (E/R).
 *  - An expert id of -1 masks the pair: no slot (slot_of_pair = -1), not
 *    counted, skipped by combine.  Ids outside [-1, E) are reported and then
 *    handled like -1.
 *  - Combine: acc = +0.0f, then acc = fmaf(w[t,j], y[slot(t,j)], acc) for
 *    j = 0..k-1 in order, output bf16 round-to-nearest-even of acc.
 *  - combine backward: grad_y[slot(t,j)] = bf16(w[t,j] * g[t]) (one fp32
 *    product, then bf16 rounding); grad_w[t,j] = sum_h g[t,h] * y[slot,h],
 *    accumulated here in double and rounded to float once.
 *  - dispatch backward: grad_x[t] = bf16(sum_j grad_recv[slot(t,j)]), fp32
 *    adds from +0.0f in j order; the gradient through FP8 quantisation is
 *    taken as the identity (straight-through).
 */
#include "ep_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- formats */

/* Value of an E4M3 code: normal codes are (1 + m/8) * 2^(e-7) = (8+m)*2^(e-10),
 * exponent field 0 gives m * 2^-9. */
double epo_e4m3_value(uint8_t code) {
  int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double mag = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
  return s ? -mag : mag;
}

/* floor(log2(a)) for a > 0 */
static int ilog2_floor(double a) {
  int e;
  frexp(a, &e); /* a = f * 2^e, f in [0.5, 1) */
  return e - 1;
}

/* Round |v| to the E4M3 grid (ties to even) and saturate; then write the
 * fields of the rounded value. */
uint8_t epo_e4m3_encode(float v) {
  uint8_t s = signbit(v) ? 0x80 : 0x00;
  double a = fabs((double)v);
  if (a > 448.0) return (uint8_t)(s | 0x7E);
  /* spacing of the grid at a: 2^-9 below 2^-6 (subnormals), else 2^(floor(log2 a) - 3) */
  double q = (a < ldexp(1.0, -6)) ? ldexp(1.0, -9) : ldexp(1.0, ilog2_floor(a) - 3);
  double r = rint(a / q) * q; /* a / q is exact; rint rounds half to even */
  if (r > 448.0) r = 448.0;
  if (r < ldexp(1.0, -6)) return (uint8_t)(s | (uint8_t)(r / ldexp(1.0, -9)));
  int ex = ilog2_floor(r);
  int m = (int)(r / ldexp(1.0, ex) * 8.0) - 8;
  return (uint8_t)(s | (uint8_t)((ex + 7) << 3) | (uint8_t)m);
}

float epo_f32_from_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* bf16 keeps 8 significant bits: round |f| to a multiple of 2^(floor(log2|f|) - 7)
 * (2^-133 in the subnormal range below 2^-126), ties to even; overflow gives inf. */
uint16_t epo_bf16_from_f32(float f) {
  uint16_t s = signbit(f) ? 0x8000 : 0x0000;
  if (isnan(f)) return (uint16_t)(s | 0x7FC0);
  if (isinf(f)) return (uint16_t)(s | 0x7F80);
  double a = fabs((double)f);
  if (a == 0.0) return s;
  double q = (a < ldexp(1.0, -126)) ? ldexp(1.0, -133) : ldexp(1.0, ilog2_floor(a) - 7);
  double r = rint(a / q) * q;
  if (r >= ldexp(1.0, 128)) return (uint16_t)(s | 0x7F80);
  float rf = (float)r; /* exact: r has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &rf, 4);
  return (uint16_t)(s | (uint16_t)(u >> 16));
}

void epo_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = epo_e4m3_encode(v[i]);
}
void epo_e4m3_value_array(const uint8_t* c, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = epo_e4m3_value(c[i]);
}
void epo_bf16_from_f32_array(const float* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = epo_bf16_from_f32(v[i]);
}

/* ----------------------------------------------------------------- layout */

int epo_layout(int64_t T, int64_t k, int64_t E, int64_t R, const int64_t* topk_idx,
               int32_t* num_tokens_per_expert, int32_t* expert_offset,
               int32_t* num_tokens_per_rank, int32_t* count_src_rank_expert,
               int32_t* src_rank_expert_offset, uint8_t* is_token_in_rank,
               int32_t* slot_of_pair, int32_t* src_of_slot) {
  if (T < 0 || k < 1 || E < 1 || R < 1 || E % R != 0 || T % R != 0) return EPO_INVALID;
  int64_t Tr = T / R, Er = E / R;
  int status = EPO_OK;

  for (int64_t e = 0; e < E; ++e) num_tokens_per_expert[e] = 0;
  for (int64_t i = 0; i < R * E; ++i) count_src_rank_expert[i] = 0;
  for (int64_t i = 0; i < T * R; ++i) is_token_in_rank[i] = 0;

  /* counts */
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t j = 0; j < k; ++j) {
      int64_t e = topk_idx[t * k + j];
      if (e == -1) continue;
      if (e < -1 || e >= E) { status = EPO_BAD_INDEX; continue; }
      num_tokens_per_expert[e] += 1;
      is_token_in_rank[t * R + e / Er] = 1;
      count_src_rank_expert[(t / Tr) * E + e] += 1;
    }
  }
  for (int64_t r = 0; r < R; ++r) {
    int32_t n = 0;
    for (int64_t t = 0; t < T; ++t) n += is_token_in_rank[t * R + r];
    num_tokens_per_rank[r] = n;
  }

  /* offsets: exclusive prefix sums */
  expert_offset[0] = 0;
  for (int64_t e = 0; e < E; ++e) expert_offset[e + 1] = expert_offset[e] + num_tokens_per_expert[e];
  for (int64_t e = 0; e < E; ++e) {
    int32_t run = expert_offset[e];
    for (int64_t r = 0; r < R; ++r) {
      src_rank_expert_offset[r * E + e] = run;
      run += count_src_rank_expert[r * E + e];
    }
  }

  /* slots: walk the pairs in (t, j) order, each expert hands out its rows in turn */
  int32_t* cursor = (int32_t*)malloc((size_t)E * sizeof(int32_t));
  for (int64_t e = 0; e < E; ++e) cursor[e] = expert_offset[e];
  for (int64_t p = 0; p < T * k; ++p) src_of_slot[p] = -1;
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t j = 0; j < k; ++j) {
      int64_t e = topk_idx[t * k + j];
      if (e < 0 || e >= E) { slot_of_pair[t * k + j] = -1; continue; }
      int32_t s = cursor[e]++;
      slot_of_pair[t * k + j] = s;
      src_of_slot[s] = (int32_t)(t * k + j);
    }
  }
  free(cursor);
  return status;
}

/* Padded layout (the low-latency kernels' static receive buffer: per local
 * expert, R blocks of M rows, one block per source rank). */
int epo_layout_padded(int64_t T, int64_t k, int64_t E, int64_t R, int64_t M, const int64_t* topk_idx,
                      int32_t* num_tokens_per_expert, int32_t* expert_offset,
                      int32_t* num_tokens_per_rank, int32_t* count_src_rank_expert,
                      int32_t* src_rank_expert_offset, uint8_t* is_token_in_rank,
                      int32_t* slot_of_pair, int32_t* src_of_row) {
  if (T < 0 || k < 1 || E < 1 || R < 1 || E % R != 0 || T % R != 0 || M < T / R || M < 1) return EPO_INVALID;
  int64_t Tr = T / R, Er = E / R;
  int status = EPO_OK;

  for (int64_t e = 0; e < E; ++e) num_tokens_per_expert[e] = 0;
  for (int64_t i = 0; i < R * E; ++i) count_src_rank_expert[i] = 0;
  for (int64_t i = 0; i < T * R; ++i) is_token_in_rank[i] = 0;
  for (int64_t i = 0; i < E * R * M; ++i) src_of_row[i] = -1;
  for (int64_t e = 0; e <= E; ++e) expert_offset[e] = (int32_t)(e * R * M);
  for (int64_t r = 0; r < R; ++r)
    for (int64_t e = 0; e < E; ++e) src_rank_expert_offset[r * E + e] = (int32_t)((e * R + r) * M);

  /* walk the pairs in (t, j) order; (source rank, expert) blocks fill in turn */
  for (int64_t t = 0; t < T; ++t) {
    int64_t r = t / Tr;
    for (int64_t j = 0; j < k; ++j) {
      int64_t e = topk_idx[t * k + j];
      slot_of_pair[t * k + j] = -1;
      if (e == -1) continue;
      if (e < -1 || e >= E) { status |= EPO_BAD_INDEX; continue; }
      num_tokens_per_expert[e] += 1;
      is_token_in_rank[t * R + e / Er] = 1;
      int64_t i = count_src_rank_expert[r * E + e]++;
      if (i >= M) { status |= EPO_CAPACITY; continue; }
      int64_t row = (e * R + r) * M + i;
      slot_of_pair[t * k + j] = (int32_t)row;
      src_of_row[row] = (int32_t)(t * k + j);
    }
  }
  for (int64_t r = 0; r < R; ++r) {
    int32_t n = 0;
    for (int64_t t = 0; t < T; ++t) n += is_token_in_rank[t * R + r];
    num_tokens_per_rank[r] = n;
  }
  return status;
}

/* ---------------------------------------------------------------- routing */

/* Group-limited gating: experts are split into groups and a token first
 * chooses groups, then experts inside them ("top-4 groups, top-8 experts":
 * "deepep-expert-parallel-communication-library", section 一 and section 三 on group-limited gating). */
int epo_route_group_limited(int64_t T, int64_t E, int64_t k, int64_t n_groups, int64_t topk_groups,
                            const float* scores, int64_t* topk_idx, float* topk_weights) {
  if (n_groups < 1 || E % n_groups != 0 || topk_groups < 1 || topk_groups > n_groups) return EPO_INVALID;
  int64_t per = E / n_groups;
  if (k < 1 || k > topk_groups * per) return EPO_INVALID;
  float* gscore = (float*)malloc((size_t)n_groups * sizeof(float));
  char* gsel = (char*)malloc((size_t)n_groups);
  char* taken = (char*)malloc((size_t)E);
  for (int64_t t = 0; t < T; ++t) {
    const float* s = scores + t * E;
    for (int64_t g = 0; g < n_groups; ++g) {
      float m = s[g * per];
      for (int64_t i = 1; i < per; ++i)
        if (s[g * per + i] > m) m = s[g * per + i];
      gscore[g] = m;
      gsel[g] = 0;
    }
    /* best groups: repeatedly the highest remaining group score, lowest index on ties */
    for (int64_t n = 0; n < topk_groups; ++n) {
      int64_t best = -1;
      for (int64_t g = 0; g < n_groups; ++g)
        if (!gsel[g] && (best < 0 || gscore[g] > gscore[best])) best = g;
      gsel[best] = 1;
    }
    /* best experts inside the chosen groups, in order */
    for (int64_t e = 0; e < E; ++e) taken[e] = 0;
    for (int64_t j = 0; j < k; ++j) {
      int64_t best = -1;
      for (int64_t e = 0; e < E; ++e)
        if (gsel[e / per] && !taken[e] && (best < 0 || s[e] > s[best])) best = e;
      taken[best] = 1;
      topk_idx[t * k + j] = best;
    }
    /* softmax of the chosen scores */
    double mx = s[topk_idx[t * k]], sum = 0.0;
    for (int64_t j = 1; j < k; ++j)
      if (s[topk_idx[t * k + j]] > mx) mx = s[topk_idx[t * k + j]];
    for (int64_t j = 0; j < k; ++j) sum += exp((double)s[topk_idx[t * k + j]] - mx);
    for (int64_t j = 0; j < k; ++j) topk_weights[t * k + j] = (float)(exp((double)s[topk_idx[t * k + j]] - mx) / sum);
  }
  free(gscore);
  free(gsel);
  free(taken);
  return EPO_OK;
}

/* --------------------------------------------------------------- dispatch */

void epo_dispatch_bf16(int64_t T, int64_t H, int64_t k, const uint16_t* x,
                       const float* topk_weights, const int32_t* slot_of_pair,
                       uint16_t* recv_x, float* recv_weight) {
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t j = 0; j < k; ++j) {
      int32_t s = slot_of_pair[t * k + j];
      if (s < 0) continue;
      for (int64_t h = 0; h < H; ++h) recv_x[(int64_t)s * H + h] = x[t * H + h];
      if (recv_weight) recv_weight[s] = topk_weights[t * k + j];
    }
  }
}

void epo_dispatch_fp8(int64_t T, int64_t H, int64_t k, const uint16_t* x,
                      const float* topk_weights, const int32_t* slot_of_pair,
                      uint8_t* recv_x, float* recv_scale, float* recv_weight) {
  int64_t G = H / 128;
  uint8_t* q = (uint8_t*)malloc((size_t)H);
  float* sc = (float*)malloc((size_t)G * sizeof(float));
  for (int64_t t = 0; t < T; ++t) {
    /* quantise the token once, per 128-channel group */
    for (int64_t g = 0; g < G; ++g) {
      float amax = 0.0f;
      for (int64_t c = 0; c < 128; ++c) {
        float a = fabsf(epo_f32_from_bf16(x[t * H + g * 128 + c]));
        if (a > amax) amax = a;
      }
      float scale = amax / 448.0f;
      if (scale == 0.0f) scale = 1.0f;
      sc[g] = scale;
      for (int64_t c = 0; c < 128; ++c) {
        float v = epo_f32_from_bf16(x[t * H + g * 128 + c]);
        q[g * 128 + c] = epo_e4m3_encode(v / scale);
      }
    }
    /* write the same payload to each of the token's slots */
    for (int64_t j = 0; j < k; ++j) {
      int32_t s = slot_of_pair[t * k + j];
      if (s < 0) continue;
      for (int64_t h = 0; h < H; ++h) recv_x[(int64_t)s * H + h] = q[h];
      for (int64_t g = 0; g < G; ++g) recv_scale[(int64_t)s * G + g] = sc[g];
      if (recv_weight) recv_weight[s] = topk_weights[t * k + j];
    }
  }
  free(q);
  free(sc);
}

/* ---------------------------------------------------------------- combine */

void epo_combine(int64_t T, int64_t H, int64_t k, const uint16_t* y,
                 const float* topk_weights, const int32_t* slot_of_pair, uint16_t* out) {
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t h = 0; h < H; ++h) {
      float acc = 0.0f;
      for (int64_t j = 0; j < k; ++j) {
        int32_t s = slot_of_pair[t * k + j];
        if (s < 0) continue;
        acc = fmaf(topk_weights[t * k + j], epo_f32_from_bf16(y[(int64_t)s * H + h]), acc);
      }
      out[t * H + h] = epo_bf16_from_f32(acc);
    }
  }
}

/* ------------------------------------------------------------- backwards */

void epo_combine_backward(int64_t T, int64_t H, int64_t k, const uint16_t* grad_out,
                          const uint16_t* y, const float* topk_weights,
                          const int32_t* slot_of_pair, uint16_t* grad_y, float* grad_w) {
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t j = 0; j < k; ++j) {
      int32_t s = slot_of_pair[t * k + j];
      if (s < 0) { grad_w[t * k + j] = 0.0f; continue; }
      float w = topk_weights[t * k + j];
      double dot = 0.0;
      for (int64_t h = 0; h < H; ++h) {
        float g = epo_f32_from_bf16(grad_out[t * H + h]);
        float prod = w * g;
        grad_y[(int64_t)s * H + h] = epo_bf16_from_f32(prod);
        dot += (double)g * (double)epo_f32_from_bf16(y[(int64_t)s * H + h]);
      }
      grad_w[t * k + j] = (float)dot;
    }
  }
}

void epo_dispatch_backward(int64_t T, int64_t H, int64_t k, const uint16_t* grad_recv,
                           const int32_t* slot_of_pair, uint16_t* grad_x) {
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t h = 0; h < H; ++h) {
      float acc = 0.0f;
      for (int64_t j = 0; j < k; ++j) {
        int32_t s = slot_of_pair[t * k + j];
        if (s < 0) continue;
        acc = acc + epo_f32_from_bf16(grad_recv[(int64_t)s * H + h]);
      }
      grad_x[t * H + h] = epo_bf16_from_f32(acc);
    }
  }
}
