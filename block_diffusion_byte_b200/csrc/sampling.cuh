// Stochastic decoding on the device: temperature / top-p draws and the
// rejection-sampling verification of drafts.
//
// Fast-BLT (discuss.pytorch.kr), "블록 언마스킹 전략": the unmasking rules can be
// combined with top-p sampling for diverse generation (which positions commit is
// decided as in the greedy rules; the committed bytes are drawn).  "BLT-S와
// BLT-DV": with a non-zero temperature the verification extends through
// rejection sampling.  The definitions (the pages give none):
//   dist = softmax(z / T) over the 256 byte logits; bytes ranked by probability
//     (ties: lower byte first); the shortest leading run reaching top_p is kept
//     and renormalised;
//   draw(dist, u) = the smallest byte b with cdf(b) > u, cdf over byte values
//     in increasing order (past the total mass: the last byte with mass);
//   verification of draft x_0..x_{k-1} drawn from q_t, with targets p_t (slot t
//     predicted by the row before it): x_t is accepted while u_t < min(1,
//     p_t(x_t) / q_t(x_t)); at the first rejection the next byte is drawn from
//     max(p_t - q_t, 0) renormalised (p_t if that is all zero) with u_{k+t}; if
//     all k are accepted, one more byte is drawn from p_k with u_{2k}.
// Random numbers are inputs (the caller's uniforms); fp32 throughout.
#pragma once

#include "kernels.cuh"

namespace bltdec {

struct SampleArgs {
  float temperature, top_p;
  const float* u;  // [batch][ustride] uniforms in [0, 1)
  int ustride;
  float* qdist;    // [batch][kMaxBlock][256]: the distribution each draft byte was drawn from
  float* p0dist;   // [batch][256]: the target of draft slot 0 (the last committed row's prediction)
  float* pdist;    // [batch][256]: scratch of the verification
};

// Compare-exchange of 64-bit keys for a descending bitonic network.
__device__ __forceinline__ void cx_desc(unsigned long long& a, unsigned long long& b, bool desc) {
  const bool sw = desc ? (a < b) : (a > b);
  if (sw) {
    const unsigned long long t = a;
    a = b;
    b = t;
  }
}

// One warp: dist[0..255] (global) = the tempered top-p distribution of logits z.
// Element i of the sort lives in lane i mod 32, register i / 32.
__device__ void warp_tempered_top_p(const float* z, float T, float top_p, float* dist, int lane) {
  float v[8];
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[j] = __ldcg(z + lane + 32 * j) / T;
    m = fmaxf(m, v[j]);
  }
  m = warp_max(m);
  float sl = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[j] = expf(v[j] - m);
    sl += v[j];
  }
  const float S = warp_sum(sl);
  unsigned long long key[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float p = v[j] / S;
    key[j] = ((unsigned long long)__float_as_uint(p) << 32) | (unsigned)(255 - (lane + 32 * j));
  }
  // bitonic sort, descending (probability, then lower byte first)
#pragma unroll
  for (int size = 2; size <= 256; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= 32) {
        const int js = stride >> 5;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if ((j & js) == 0) cx_desc(key[j], key[j | js], ((lane + 32 * j) & size) == 0);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = lane + 32 * j;
          const unsigned long long o = __shfl_xor_sync(0xffffffffu, key[j], stride);
          const bool desc = (i & size) == 0;
          const bool lower = (i & stride) == 0;
          // the lower index of a pair keeps the larger key in a descending block
          const bool take_max = (lower == desc);
          key[j] = take_max ? (key[j] > o ? key[j] : o) : (key[j] < o ? key[j] : o);
        }
      }
    }
  }
  // inclusive prefix sums in sorted order; the cut n = first index reaching top_p
  float cum[8];
  float carry = 0.f;
  int n = 256;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float c = __uint_as_float((unsigned)(key[j] >> 32));
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float t = __shfl_up_sync(0xffffffffu, c, o);
      if (lane >= o) c += t;
    }
    cum[j] = carry + c;
    carry += __shfl_sync(0xffffffffu, c, 31);
    const unsigned hit = __ballot_sync(0xffffffffu, cum[j] >= top_p);
    if (hit && n == 256) n = 32 * j + __ffs(hit) - 1;
  }
  if (n == 256) n = 255;  // rounding left the total short of top_p: keep everything
  const float kept = __shfl_sync(0xffffffffu, cum[n >> 5], n & 31);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = lane + 32 * j;
    const int b = 255 - (int)(key[j] & 0xFFu);
    dist[b] = (i <= n) ? __uint_as_float((unsigned)(key[j] >> 32)) / kept : 0.f;
  }
  __threadfence_block();  // the warp reads dist next (after __syncwarp)
}

// One warp: the byte drawn from dist (global, 256) with uniform u.
__device__ int warp_draw(const float* dist, float u, int lane) {
  float d[8], pre[8];
  float run = 0.f;
  int last = -1;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    d[j] = __ldcg(dist + 8 * lane + j);
    run += d[j];
    pre[j] = run;
    if (d[j] > 0.f) last = 8 * lane + j;
  }
  float base = run;  // exclusive scan of the lanes' totals
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float t = __shfl_up_sync(0xffffffffu, base, o);
    if (lane >= o) base += t;
  }
  base -= run;
  int cand = 256;
#pragma unroll
  for (int j = 7; j >= 0; --j)
    if (d[j] > 0.f && base + pre[j] > u) cand = 8 * lane + j;
  int best = cand;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = min(best, __shfl_xor_sync(0xffffffffu, best, o));
  if (best < 256) return best;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
  return max(last, 0);
}

// Verification of sequence s's k draft bytes by rejection sampling (one warp).
// Target of slot t: p0dist for t = 0, else the verification row t - 1.
__device__ void accept_seq_sampled(SeqDev sd, int s, int k, const SampleArgs& sa, const int* vlat, const float* logits,
                                   int* out_acc, unsigned char* out_next, float* out_logits, int lane) {
  const float* us = sa.u + (size_t)s * sa.ustride;
  float* pd = sa.pdist + (size_t)s * 256;
  int a = k, nxt = 0;
  for (int t = 0; t < k; ++t) {
    const float* pt;
    if (t == 0) {
      pt = sa.p0dist + (size_t)s * 256;
    } else {
      warp_tempered_top_p(logits + (size_t)sd.blk_row[s * kMaxBlock + t - 1] * 256, sa.temperature, sa.top_p, pd, lane);
      __syncwarp();
      pt = pd;
    }
    const float* qt = sa.qdist + ((size_t)s * kMaxBlock + t) * 256;
    const int x = sd.blk[s * kMaxBlock + t];
    const float qx = __ldcg(qt + x), px = __ldcg(pt + x);
    const float ratio = qx > 0.f ? fminf(1.f, px / qx) : 1.f;
    if (__ldcg(us + t) < ratio) continue;
    // rejected: the residual max(p - q, 0), renormalised, into pd
    float r[8];
    float rs = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int b = lane + 32 * j;
      r[j] = fmaxf(__ldcg(pt + b) - __ldcg(qt + b), 0.f);
      rs += r[j];
    }
    rs = warp_sum(rs);
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int b = lane + 32 * j;
      pd[b] = rs > 0.f ? r[j] / rs : __ldcg(pt + b);
    }
    __threadfence_block();
    __syncwarp();
    a = t;
    nxt = warp_draw(pd, __ldcg(us + k + t), lane);
    break;
  }
  if (a == k) {
    warp_tempered_top_p(logits + (size_t)sd.blk_row[s * kMaxBlock + k - 1] * 256, sa.temperature, sa.top_p, pd, lane);
    __syncwarp();
    nxt = warp_draw(pd, __ldcg(us + 2 * k), lane);
  }
  if (out_logits && lane < k) {
    const int row = sd.blk_row[s * kMaxBlock + lane];
    float* dst = out_logits + ((size_t)s * k + lane) * 256;
    for (int j = 0; j < 256; ++j) dst[j] = __ldcg(logits + (size_t)row * 256 + j);
  }
  if (lane == 0) {
    out_acc[s] = a;
    out_next[s] = (unsigned char)nxt;
    sd.kv_len[s] += a;
    if (a >= 1) sd.n_lat[s] = max(sd.n_lat[s], vlat[s * k + a - 1] + 1);
  }
}

__global__ void k_accept_sampled(SeqDev sd, int batch, int k, SampleArgs sa, const int* vlat, const float* logits, int* out_acc,
                                 unsigned char* out_next, float* out_logits) {
  const int s = blockIdx.x;
  if (s < batch) accept_seq_sampled(sd, s, k, sa, vlat, logits, out_acc, out_next, out_logits, threadIdx.x & 31);
}

// The draft byte of AR drafting step `step` drawn from its row's distribution.
__global__ void k_draft_ar_sampled(SeqDev sd, int batch, int step, SampleArgs sa, const int* pred, const float* logits,
                                   float* out_logits) {
  const int s = blockIdx.x, lane = threadIdx.x & 31;
  if (s >= batch) return;
  const int row = (step == 0) ? sd.last_row[s] : sd.blk_row[s * kMaxBlock];
  float* q = sa.qdist + ((size_t)s * kMaxBlock + step) * 256;
  warp_tempered_top_p(logits + (size_t)row * 256, sa.temperature, sa.top_p, q, lane);
  __syncwarp();
  const int b = warp_draw(q, __ldcg(sa.u + (size_t)s * sa.ustride + step), lane);
  if (step == 0)  // slot 0's draft and target are the same row's prediction
    for (int j = lane; j < 256; j += 32) sa.p0dist[(size_t)s * 256 + j] = __ldcg(q + j);
  if (lane == 0) {
    sd.blk[s * kMaxBlock + step] = (unsigned char)b;
    if (step == 0) sd.y_last[s] = __ldcg(pred + row);
  }
  if (out_logits)
    for (int j = lane; j < 256; j += 32) out_logits[((size_t)step * batch + s) * 256 + j] = __ldcg(logits + (size_t)row * 256 + j);
}

// The bytes of the positions unmask_seq committed in this pass (bits of `newly`),
// drawn from their rows' distributions; in the first pass also slot 0's target.
__device__ void draw_committed(SeqDev sd, int s, int step, unsigned newly, const SampleArgs& sa, const float* logits, int lane) {
  if (step == 0) {
    const int lr = sd.last_row[s];
    if (lr >= 0) warp_tempered_top_p(logits + (size_t)lr * 256, sa.temperature, sa.top_p, sa.p0dist + (size_t)s * 256, lane);
  }
  while (newly) {
    const int i = __ffs(newly) - 1;
    newly &= newly - 1;
    float* q = sa.qdist + ((size_t)s * kMaxBlock + i) * 256;
    warp_tempered_top_p(logits + (size_t)sd.blk_row[s * kMaxBlock + i] * 256, sa.temperature, sa.top_p, q, lane);
    __syncwarp();
    const int b = warp_draw(q, __ldcg(sa.u + (size_t)s * sa.ustride + i), lane);
    if (lane == 0) sd.blk[s * kMaxBlock + i] = (unsigned char)b;
    __syncwarp();
  }
}

// unmask_seq's selection, then the committed positions' bytes drawn (one warp per sequence).
__global__ void k_unmask_sampled(SeqDev sd, int batch, int k, float alpha, int step, SampleArgs sa, const float* conf,
                                 const int* pred, const float* logits, float* out_logits, const float* ent) {
  const int s = blockIdx.x, lane = threadIdx.x & 31;
  if (s >= batch || !sd.active[s]) return;
  unsigned newly = 0;
  unmask_seq(sd, s, batch, k, alpha, step, conf, pred, logits, out_logits, lane, ent, &newly, false);
  __syncwarp();
  draw_committed(sd, s, step, newly, sa, logits, lane);
}

}  // namespace bltdec
