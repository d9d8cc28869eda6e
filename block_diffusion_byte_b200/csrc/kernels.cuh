// Kernels of the Fast-BLT local-decoder pass and its bookkeeping (sm_100a).
//
// Decoder layer (the layer equation of "Fast Byte Latent Transformer
// (Fast-BLT) 연구 소개", section "계층적 BLT: 인코더, 글로벌 모델, 디코더"):
//   B_l = D_{l-1} + W_o^c softmax(Q K^T / sqrt(d_k)) V     (cross-attention)
//   D_l = DecoderTransformerLayer(B_l)                     (pre-norm self-attn + SwiGLU)
// A row sees exactly one latent o (section "BLT-D의 어텐션 마스크"), so the
// softmax is exactly 1 and the cross term is c = W_o^c W_v^c o, projected once
// when the latent arrives and gathered per row.
//
// Canonical arithmetic of every projection y = rs * (W (g . x)):
//   x is the fp32 input row, g the RMSNorm gain (1 when there is no norm),
//   g . x is split into bf16 planes hi + lo; W is one bf16 plane (two for
//   fp32 weights).  K is cut into k16 steps; step s belongs to lane group
//   w = s mod 8, which accumulates in increasing s the tensor-core products
//   W_hi x_hi, W_hi x_lo (, W_lo x_hi) into one fp32 accumulator.  The output
//   is rs * (((a_0 + a_1) + ...) + a_7).  The RMS scale rs = 1/sqrt(ss/K + eps)
//   takes ss from the same fragments: every lane adds x^2 of its four values in
//   k order, the four lanes of a row are summed by xor-shuffles (1 then 2) and
//   the eight groups in order.  K beyond 1024 is cut into segments of 1024
//   columns (64 k-steps): each segment is reduced as above, and the segment
//   sums are added in order, ((S_0 + S_1) + S_2) + ..., before the scale.
//   Nothing depends on which other rows share the pass, or on which kernel
//   (per-phase or persistent) runs it, so a row's results are bit-identical
//   in every pass shape.
#pragma once

#include "common.cuh"

namespace bltdec {

// ------------------------------------------------------------------------ shared state
struct RowsDev {  // per-pass row metadata (arrays of max_rows; counts are device scalars)
  int* seq;       // sequence of the row
  int* pos;       // 0-based byte position (RoPE, KV slot)
  int* lat;       // latent slot seen by the cross-attention
  int* nkeys;     // the row attends positions 0 .. nkeys-1 of its sequence
  int* byte;      // input id (0..255 or [MASK])
  int* n_rows;    // device scalar
  int* g_seq;     // attention groups: up to 32 consecutive rows of one sequence
  int* g_row0;
  int* g_nrows;
  int* g_kmax;
  int* g_fresh;   // first position written by this pass in the group's sequence
  int* n_groups;  // device scalar
};

constexpr int kMaxCallBatch = 256;
constexpr int kSegCols = 1024;  // canonical K segment (columns)

struct CallDesc {  // by value as a kernel parameter
  int batch;
  int row_off[kMaxCallBatch + 1];
  int lat_off[kMaxCallBatch + 1];
};

struct SeqDev {
  int* kv_len;      // cached committed positions
  int* kv_base;     // kv_len at call start (prefill)
  int* n_lat;       // committed latent slots
  int* active;      // block still has masked positions
  int* steps;       // passes used by the current block
  int* y_last;      // greedy prediction of the last pending row (verification y_l)
  int* last_row;    // row index of the last pending row in pass 1 (-1: none)
  int* blk_row;     // [batch][kMaxBlock] row index of block/draft/verify row i in this pass
  unsigned char* blk;     // [batch][kMaxBlock] block / draft bytes
  unsigned char* masked;  // [batch][kMaxBlock]
  int* status;
  unsigned long long* counters;  // passes, rows, prefill_rows, latents, calls, weight_bytes, kv_bytes (decoder passes), kv_bytes (prefill)
};

enum PlanMode : int { PL_PREFILL = 0, PL_FIRST = 1, PL_BLOCK = 2, PL_ARDRAFT = 3, PL_VERIFY = 4 };

struct PlanArgs {
  int mode, k, step, r0, r1;
  int max_ctx, max_lat, mask_id;
  const unsigned char* pend_bytes;
  const int* pend_lat;
  const int* vlat;  // verify slots [batch][k]
  unsigned long long weight_bytes_per_pass;
  unsigned long long kv_bytes_per_key;
};

// ------------------------------------------------------------------------ GEMM pieces
enum Epi : int { EPI_STORE = 0, EPI_RESID = 1, EPI_SWIGLU = 2, EPI_QKV = 3, EPI_LATC = 4, EPI_XRESID = 5 };

struct GemmArgs {
  const uint4* w;  // tiles [N/16][K/16][planes][32 lanes] of 16 B
  int N, K;
  const float* X;  // activations [rows][ldx] fp32
  int ldx;
  int group_tiles, group_xoff;  // if group_tiles > 0: output tile mt reads X + (mt / group_tiles) * group_xoff
  const float* gain;  // [K] RMSNorm gain; NULL: no norm (rs = 1)
  float eps;
  const int* n_rows;  // device row count (NULL: rows_host is exact)
  int rows_host;
  float* out;  // EPI_STORE / RESID / SWIGLU / LATC / XRESID base
  int ldo;
  // EPI_XRESID: out = (xsrc + c_lat) + v, xsrc = embed[byte] in layer 0, else out itself
  const float* embed;
  const float* c_lat;
  // EPI_QKV
  float* q;
  void* kv;  // KV pool: bf16, or fp32 when kv_f32
  int kv_f32;
  const int* page_table;
  int max_pages, PT, layer, L, H, dh, d;
  const int* row_seq;
  const int* row_pos;
  const int* row_lat;
  const int* row_byte;
  const float* rope_cos;  // [max_ctx][dh/2], or [row][dh/2] when rope_by_row
  const float* rope_sin;
  int rope_by_row;      // rope tables indexed by activation row (per-pass copy) instead of position
  const int* row_page;  // KV page of each row's position (-1: none); NULL: look up page_table
  // EPI_LATC
  const int* lat_seq;
  const int* lat_slot;
  int max_lat;
  int* status;
  // split over K segments (K > kSegCols, no gain): CTA z computes segment z's sums into
  // seg_ws [nseg][seg_rows][N]; k_seg_finish adds them in order and runs the epilogue
  float* seg_ws;
  int seg_rows;
};

// Four gained values of one k16 step -> hi/lo B fragments (k = 2t, 2t+1 | 2t+8, 2t+9).
struct XFrag {
  uint32_t b0h, b1h, b0l, b1l;
};
__device__ __forceinline__ XFrag make_xfrag(float x0, float x1, float x8, float x9) {
  XFrag f;
  split2(x0, x1, f.b0h, f.b0l);
  split2(x8, x9, f.b1h, f.b1l);
  return f;
}
__device__ __forceinline__ float ss_add(float ss, float v0, float v1, float v8, float v9) {
  ss = fmaf(v0, v0, ss);
  ss = fmaf(v1, v1, ss);
  ss = fmaf(v8, v8, ss);
  return fmaf(v9, v9, ss);
}
template <int PL>
__device__ __forceinline__ void mma_step(float (&c)[4], const uint4 (&w)[PL], const XFrag& x) {
  mma16816(c, w[0], x.b0h, x.b1h);
  mma16816(c, w[0], x.b0l, x.b1l);
  if constexpr (PL == 2) mma16816(c, w[1], x.b0h, x.b1h);
}

// Element offset of (page, layer, K|V, head, position in page, dim) in the KV pool.
// K/V rows of 64 bf16 (128 bytes) are stored with their 16-byte pieces permuted by
// position: piece j of position pos sits at piece j ^ (pos mod 8).  A chunk copied as
// is into shared memory (128-key chunks start at multiples of 8) then has the eight
// rows of every 8x8 ldmatrix tile in eight different bank groups.  Other K/V formats
// are stored plainly.
__device__ __forceinline__ int kv_dim(const GemmArgs& a, int pos, int dim) {
  return (a.kv_f32 || a.dh != 64) ? dim : ((((dim >> 3) ^ pos) & 7) << 3) | (dim & 7);
}
__device__ __forceinline__ size_t kv_offset(const GemmArgs& a, int page, int layer, int kvsel, int h, int off, int dim) {
  return ((((size_t)page * a.L + layer) * 2 + kvsel) * a.H + h) * (size_t)a.PT * a.dh + (size_t)off * a.dh + dim;
}

__device__ __forceinline__ const float* c_row(const float* c_lat, int max_lat, int L, int layer, int d, int seq, int lat) {
  return c_lat + (((size_t)seq * max_lat + lat) * L + layer) * d;
}

__device__ __forceinline__ void kv_store(const GemmArgs& a, size_t off, float v) {
  if (a.kv_f32) static_cast<float*>(a.kv)[off] = v;
  else static_cast<__nv_bfloat16*>(a.kv)[off] = __float2bfloat16_rn(v);
}

// KV page holding position `pos` of `seq` (-1: not allocated).
__device__ __forceinline__ int row_kv_page(const GemmArgs& a, int row, int seq, int pos) {
  if (a.row_page) return a.row_page[row];
  const int pi = pos / a.PT;
  return (pi < a.max_pages) ? a.page_table[seq * a.max_pages + pi] : -1;
}

// Output pair of tile rows (r16, r16 + 8) of tile mt for activation row `row`.
// Row metadata pointers may point to shared memory (persistent kernel copies).
template <int EPI>
__device__ __forceinline__ void gemm_epilogue(const GemmArgs& a, int mt, int r16, int row, float v0, float v1) {
  if constexpr (EPI == EPI_STORE) {
    float* o = a.out + (size_t)row * a.ldo + mt * 16 + r16;
    o[0] = v0;
    o[8] = v1;
  } else if constexpr (EPI == EPI_RESID) {
    float* o = a.out + (size_t)row * a.ldo + mt * 16 + r16;
    o[0] = __ldcg(o) + v0;
    o[8] = __ldcg(o + 8) + v1;
  } else if constexpr (EPI == EPI_XRESID) {
    const int n = mt * 16 + r16;
    const float* src = (a.layer == 0) ? a.embed + (size_t)a.row_byte[row] * a.d : a.out + (size_t)row * a.ldo;
    const float* c = c_row(a.c_lat, a.max_lat, a.L, a.layer, a.d, a.row_seq[row], a.row_lat[row]);
    const float s0 = __ldcg(src + n) + __ldcg(c + n), s1 = __ldcg(src + n + 8) + __ldcg(c + n + 8);
    float* o = a.out + (size_t)row * a.ldo + n;
    o[0] = s0 + v0;
    o[8] = s1 + v1;
  } else if constexpr (EPI == EPI_SWIGLU) {
    a.out[(size_t)row * a.ldo + mt * 8 + r16] = silu(v0) * v1;
  } else if constexpr (EPI == EPI_LATC) {
    float* o = a.out + (((size_t)a.lat_seq[row] * a.max_lat + a.lat_slot[row]) * a.L + a.layer) * a.d + mt * 16 + r16;
    o[0] = v0;
    o[8] = v1;
  } else {  // EPI_QKV: q/k tiles hold rotary pairs (j, j + dh/2) in rows (r16, r16 + 8)
    const int tiles_sec = a.d / 16;
    const int sec = mt / tiles_sec, lt = mt % tiles_sec;
    const int pos = a.row_pos[row];
    const int seq = a.row_seq[row];
    if (sec == 0 || sec == 1) {
      const int tph = a.dh / 16;
      const int h = lt / tph, j = (lt % tph) * 8 + r16;
      const int half = a.dh / 2;
      const size_t ri = (size_t)(a.rope_by_row ? row : pos) * half + j;
      const float c = a.rope_cos[ri], s = a.rope_sin[ri];
      const float o0 = v0 * c - v1 * s, o1 = v1 * c + v0 * s;
      if (sec == 0) {
        float* q = a.q + (size_t)row * a.d + h * a.dh;
        q[j] = o0;
        q[j + half] = o1;
        return;
      }
      const int page = row_kv_page(a, row, seq, pos);
      if (page < 0) {
        set_status(a.status, kErrDevice);
        return;
      }
      kv_store(a, kv_offset(a, page, a.layer, 0, h, pos % a.PT, kv_dim(a, pos, j)), o0);
      kv_store(a, kv_offset(a, page, a.layer, 0, h, pos % a.PT, kv_dim(a, pos, j + half)), o1);
    } else {
      const int page = row_kv_page(a, row, seq, pos);
      if (page < 0) {
        set_status(a.status, kErrDevice);
        return;
      }
      const int n0 = lt * 16 + r16, n1 = n0 + 8;
      kv_store(a, kv_offset(a, page, a.layer, 1, n0 / a.dh, pos % a.PT, kv_dim(a, pos, n0 % a.dh)), v0);
      kv_store(a, kv_offset(a, page, a.layer, 1, n1 / a.dh, pos % a.PT, kv_dim(a, pos, n1 % a.dh)), v1);
    }
  }
}

// Canonical cross-warp reduction of one tile (RB rows).  acc: each warp's
// accumulators; ss: each warp's per-lane sum of squares for row n*8+g.
// red: smem [8][16][RB]; ssr: smem [8][RB].  Calls epi(r16, col, v0, v1) with
// the scaled pair for every valid column.  `sync` is a consumer-wide barrier;
// red/ssr are free again after the call returns and the caller syncs.
template <int NG, class Sync, class Fn>
__device__ __forceinline__ void tile_reduce(const float (&acc)[NG][4], const float (&ss)[NG], bool want_ss, float* red,
                                            float* ssr, int nr, int K, float eps, int tid, int nthreads, Sync sync, Fn epi) {
  constexpr int RB = 8 * NG;
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int n = 0; n < NG; ++n) {
    const int c = n * 8 + 2 * t;
    red[(warp * 16 + g) * RB + c] = acc[n][0];
    red[(warp * 16 + g) * RB + c + 1] = acc[n][1];
    red[(warp * 16 + g + 8) * RB + c] = acc[n][2];
    red[(warp * 16 + g + 8) * RB + c + 1] = acc[n][3];
    if (want_ss) {
      float s = ss[n];
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (t == 0) ssr[warp * RB + n * 8 + g] = s;
    }
  }
  sync();
  for (int p = tid; p < 8 * RB; p += nthreads) {
    const int r16 = p & 7, col = p >> 3;
    if (col >= nr) continue;
    float v0 = red[r16 * RB + col], v1 = red[(r16 + 8) * RB + col];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
      v0 += red[(w * 16 + r16) * RB + col];
      v1 += red[(w * 16 + r16 + 8) * RB + col];
    }
    float rs = 1.0f;
    if (want_ss) {
      float s = ssr[col];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) s += ssr[w * RB + col];
      rs = 1.0f / sqrtf(s / (float)K + eps);
    }
    epi(r16, col, v0 * rs, v1 * rs);
  }
}

// K segments (K > 1024): fold a finished segment into the running totals.
// Every warp's accumulators go to red [8][16][RB]; each thread sums its output
// pairs (p = tid, tid + 256) over the warps in order -- the segment sum S_j --
// and adds it to its totals (the first segment is taken as is); accumulators
// restart at zero.  red must not alias the activation staging.
template <int NG>
__device__ __forceinline__ void seg_fold(float (&acc)[NG][4], float* red, float (&tot)[2][2], int& nsegs_done, int tid) {
  constexpr int RB = 8 * NG;
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int n = 0; n < NG; ++n) {
    const int c = n * 8 + 2 * t;
    red[(warp * 16 + g) * RB + c] = acc[n][0];
    red[(warp * 16 + g) * RB + c + 1] = acc[n][1];
    red[(warp * 16 + g + 8) * RB + c] = acc[n][2];
    red[(warp * 16 + g + 8) * RB + c + 1] = acc[n][3];
    acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int p = tid + i * kThreads;
    if (p < 8 * RB) {
      const int r16 = p & 7, col = p >> 3;
      float v0 = red[r16 * RB + col], v1 = red[(r16 + 8) * RB + col];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) {
        v0 += red[(w * 16 + r16) * RB + col];
        v1 += red[(w * 16 + r16 + 8) * RB + col];
      }
      tot[i][0] = nsegs_done ? tot[i][0] + v0 : v0;
      tot[i][1] = nsegs_done ? tot[i][1] + v1 : v1;
    }
  }
  ++nsegs_done;
  __syncthreads();
}

// After the last seg_fold: the RMS scale (if any) and the epilogue of every pair.
template <int NG, class Fn>
__device__ __forceinline__ void tile_reduce_totals(const float (&tot)[2][2], const float (&ss)[NG], bool want_ss, float* red, float* ssr,
                                                   int nr, int K, float eps, int tid, Fn epi) {
  constexpr int RB = 8 * NG;
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  if (want_ss) {
#pragma unroll
    for (int n = 0; n < NG; ++n) {
      float s = ss[n];
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (t == 0) ssr[warp * RB + n * 8 + g] = s;
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int p = tid + i * kThreads;
    if (p < 8 * RB) {
      const int r16 = p & 7, col = p >> 3;
      if (col >= nr) continue;
      float rs = 1.0f;
      if (want_ss) {
        float s = ssr[col];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) s += ssr[w * RB + col];
        rs = 1.0f / sqrtf(s / (float)K + eps);
      }
      epi(r16, col, tot[i][0] * rs, tot[i][1] * rs);
    }
  }
  (void)red;
}

// Per-phase GEMM kernel (passes with many rows, latent projection, prefill).
// One CTA: one 16-row tile of W against RB = 8*NG rows.
template <int NG, int PL, int EPI, int STAGES>
__global__ void __launch_bounds__(kThreads) k_gemm(GemmArgs a) {
  constexpr int RB = 8 * NG;
  const int nrows = a.n_rows ? *a.n_rows : a.rows_host;
  const int mt = blockIdx.x;
  const int row0 = blockIdx.y * RB;
  if (row0 >= nrows) return;
  const int nr = min(RB, nrows - row0);

  extern __shared__ float4 smem4[];
  float* xs = reinterpret_cast<float*>(smem4);  // [STAGES][RB][kXStride]
  float* ssr = xs + STAGES * RB * kXStride;     // [8][RB]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int ksteps = a.K / 16;
  const bool norm = a.gain != nullptr;
  constexpr int kSegWin = kSegCols / kKWin;  // windows per segment (a multiple of DEPTH)
  // windows [w0, nwin): all of K, or (split) segment blockIdx.z only
  const bool split = a.seg_ws != nullptr;
  const int w0 = split ? (int)blockIdx.z * kSegWin : 0;
  const int nwin = split ? w0 + kSegWin : a.K / kKWin;

  const float* xg = a.X + (a.group_tiles ? (size_t)(mt / a.group_tiles) * a.group_xoff : 0);
  auto stage = [&](int wi, int buf) {
    for (int c = tid; c < RB * 32; c += kThreads) {
      const int r = c >> 5, q = c & 31;
      const bool ok = r < nr;
      const float* src = xg + (size_t)(ok ? row0 + r : row0) * a.ldx + wi * kKWin + q * 4;
      cp_async16(xs + ((size_t)buf * RB + r) * kXStride + q * 4, src, ok ? 16 : 0);
    }
  };
  const uint4* wbase = a.w + (size_t)mt * ksteps * PL * 32 + lane;
  const uint64_t wpol = l2_evict_first();
  auto wtile = [&](int wi, int p) -> uint4 { return ldg_stream(wbase + ((size_t)(wi * kWarps + warp) * PL + p) * 32, wpol); };

  constexpr int DEPTH = 4;
  uint4 wb[DEPTH][PL];
#pragma unroll
  for (int dd = 0; dd < DEPTH; ++dd)
#pragma unroll
    for (int p = 0; p < PL; ++p) wb[dd][p] = (w0 + dd < nwin) ? wtile(w0 + dd, p) : make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (w0 + s < nwin) stage(w0 + s, (w0 + s) % STAGES);
    cp_async_commit();
  }
  float acc[NG][4], ss[NG];
#pragma unroll
  for (int n = 0; n < NG; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = ss[n] = 0.f;
  float tot[2][2] = {{0.f, 0.f}, {0.f, 0.f}};  // K > 1024: this thread's output pairs, segments summed in order
  int nsegs_done = 0;

  for (int wi0 = w0; wi0 < nwin; wi0 += DEPTH) {
    if (wi0 > w0 && wi0 % kSegWin == 0) {  // segment boundary: fold the finished segment
      seg_fold<NG>(acc, xs + (size_t)STAGES * RB * kXStride + 8 * RB, tot, nsegs_done, tid);
    }
#pragma unroll
    for (int dd = 0; dd < DEPTH; ++dd) {
      const int wi = wi0 + dd;
      if (wi < nwin) {
        uint4 wcur[PL];
#pragma unroll
        for (int p = 0; p < PL; ++p) {
          wcur[p] = wb[dd][p];
          if (wi + DEPTH < nwin) wb[dd][p] = wtile(wi + DEPTH, p);
        }
        cp_async_wait<STAGES - 2>();
        __syncthreads();
        if (wi + STAGES - 1 < nwin) stage(wi + STAGES - 1, (wi + STAGES - 1) % STAGES);
        cp_async_commit();
        const float* xw = xs + (size_t)(wi % STAGES) * RB * kXStride;
        const int kk = warp * 16 + 2 * t;
        const int kg = wi * kKWin + kk;
        float g0 = 1.f, g1 = 1.f, g8 = 1.f, g9 = 1.f;
        if (norm) {
          g0 = __ldg(a.gain + kg);
          g1 = __ldg(a.gain + kg + 1);
          g8 = __ldg(a.gain + kg + 8);
          g9 = __ldg(a.gain + kg + 9);
        }
#pragma unroll
        for (int n = 0; n < NG; ++n) {
          const float* xr = xw + (n * 8 + g) * kXStride + kk;
          const float2 p0 = *reinterpret_cast<const float2*>(xr);
          const float2 p8 = *reinterpret_cast<const float2*>(xr + 8);
          if (norm) ss[n] = ss_add(ss[n], p0.x, p0.y, p8.x, p8.y);
          mma_step<PL>(acc[n], wcur, make_xfrag(p0.x * g0, p0.y * g1, p8.x * g8, p8.y * g9));
        }
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  if (split) {  // this segment's sums S_z (the warps added in order), for k_seg_finish
    seg_fold<NG>(acc, xs, tot, nsegs_done, tid);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int p = tid + i * kThreads;
      if (p < 8 * RB) {
        const int r16 = p & 7, col = p >> 3;
        if (col < nr) {
          float* w = a.seg_ws + ((size_t)blockIdx.z * a.seg_rows + row0 + col) * a.N + mt * 16 + r16;
          w[0] = tot[i][0];
          w[8] = tot[i][1];
        }
      }
    }
    return;
  }
  if (a.K <= kSegCols) {
    tile_reduce<NG>(acc, ss, norm, xs, ssr, nr, a.K, a.eps, tid, kThreads, [] { __syncthreads(); },
                    [&](int r16, int col, float v0, float v1) { gemm_epilogue<EPI>(a, mt, r16, row0 + col, v0, v1); });
    return;
  }
  // last segment, then the ordered segment sum and the scale
  seg_fold<NG>(acc, xs, tot, nsegs_done, tid);
  tile_reduce_totals<NG>(tot, ss, norm, xs, ssr, nr, a.K, a.eps, tid,
                         [&](int r16, int col, float v0, float v1) { gemm_epilogue<EPI>(a, mt, r16, row0 + col, v0, v1); });
}

// After a split k_gemm: the segment sums added in order, ((S_0 + S_1) + S_2) + ...,
// exactly as k_gemm folds them, then the epilogue.  One thread per output pair.
template <int EPI>
__global__ void k_seg_finish(GemmArgs a, int nseg) {
  const int nrows = a.n_rows ? *a.n_rows : a.rows_host;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;  // (row, tile, r16)
  const int pairs = a.N / 2;
  const int row = i / pairs, q = i % pairs, mt = q / 8, r16 = q % 8;
  if (row >= nrows) return;
  const float* w = a.seg_ws + (size_t)row * a.N + mt * 16 + r16;
  const size_t zs = (size_t)a.seg_rows * a.N;
  float v0 = w[0], v1 = w[8];
  for (int z = 1; z < nseg; ++z) {
    v0 = v0 + w[z * zs];
    v1 = v1 + w[z * zs + 8];
  }
  gemm_epilogue<EPI>(a, mt, r16, row, v0, v1);
}

// ------------------------------------------------------------------------ row-wise kernels
// h[row] = embed[byte[row]]
__global__ void k_embed(const RowsDev rows, const float* __restrict__ embed, float* __restrict__ h, int d) {
  const int n = *rows.n_rows;
  for (int r = blockIdx.x; r < n; r += gridDim.x) {
    const float* e = embed + (size_t)rows.byte[r] * d;
    for (int i = threadIdx.x; i < d; i += blockDim.x) h[(size_t)r * d + i] = e[i];
  }
}

// h[row] += c_lat[seq][lat][layer]: the cross-attention term of the layer.
__global__ void k_cross_add(const RowsDev rows, float* __restrict__ h, const float* __restrict__ c_lat, int max_lat, int L,
                            int layer, int d) {
  const int n = *rows.n_rows;
  for (int r = blockIdx.x; r < n; r += gridDim.x) {
    const float* c = c_row(c_lat, max_lat, L, layer, d, rows.seq[r], rows.lat[r]);
    for (int i = threadIdx.x; i < d; i += blockDim.x) h[(size_t)r * d + i] += c[i];
  }
}

// ------------------------------------------------------------------------ attention
struct AttnArgs {
  const float* q;  // [rows][d], RoPE applied
  const void* kv;
  const int* page_table;
  int max_pages, PT, L, layer, H, dh, d;
  RowsDev rows;
  int CH, CMAX;
  float scale;
  float2* part_ml;  // [rows][H][CMAX]
  float* part_o;    // [rows][H][CMAX][dh]
  float* att;       // [rows][d]
  int* status;
};

constexpr int kAttnRows = 32;  // rows per attention group

__device__ __forceinline__ void widen8(const __nv_bfloat16* p, float* out) {
  const uint4 raw = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
  for (int e = 0; e < 8; ++e) out[e] = __bfloat162float(b[e]);
}
__device__ __forceinline__ void widen8(const float* p, float* out) {
  const float4 x = reinterpret_cast<const float4*>(p)[0], y = reinterpret_cast<const float4*>(p)[1];
  out[0] = x.x, out[1] = x.y, out[2] = x.z, out[3] = x.w, out[4] = y.x, out[5] = y.y, out[6] = y.z, out[7] = y.w;
}

template <int DH, typename KVT>
__device__ __forceinline__ const KVT* kv_chunk_src(const AttnArgs& a, int seq, int h, int tpos, int kvsel) {
  int page = a.page_table[seq * a.max_pages + tpos / a.PT];
  if (page < 0) {
    set_status(a.status, kErrDevice);
    page = 0;
  }
  return static_cast<const KVT*>(a.kv) + ((((size_t)page * a.L + a.layer) * 2 + kvsel) * a.H + h) * (size_t)a.PT * DH +
         (size_t)(tpos % a.PT) * DH;
}

// Row stride (elements) of a K/V chunk in shared memory: 16 bytes of padding
// so the 16-byte segments of consecutive keys fall in different banks.
template <int DH, typename KVT>
__host__ __device__ constexpr int kv_stride() {
  return DH + 16 / (int)sizeof(KVT);
}
// Whether K/V rows are stored with permuted 16-byte pieces (see kv_dim).
template <int DH, typename KVT>
__host__ __device__ constexpr bool kv_swizzled() {
  return DH == 64 && sizeof(KVT) == 2;
}
// Element (row, col) of a K/V chunk in shared memory.  ST > 0: rows of ST elements,
// plain.  ST == 0: rows of 64 elements as stored (piece j of row r at j ^ (r mod 8);
// the chunk starts at a position that is a multiple of 8).
template <int ST>
__device__ __forceinline__ int kv_at(int row, int col) {
  if constexpr (ST == 0) return row * 64 + ((((col >> 3) ^ row) & 7) << 3) + (col & 7);
  else return row * ST + col;
}

// Copy positions [lo, hi) of the chunk starting at t0 of (seq, head) into smem
// ks/vs (raw KVT, [CH][kv_stride]) with 16-byte cp.async (L2 only).  One
// K or V row per iteration: a single page-table lookup per row.
// Keys and values t0 .. t0 + n - 1 of (seq, head h) into smem (row stride ST,
// kv_stride by default), with the chunk's page ids already in pg[] (pg[j]: the page of
// positions (t0 / PT + j) PT ..): every copy is issued at once.
template <int DH, typename KVT, int ST = kv_stride<DH, KVT>()>
__device__ __forceinline__ void attn_load_kv_paged(const AttnArgs& a, const int* pg, int h, int t0, int n, KVT* ks, KVT* vs, int tid,
                                                   int nthr) {
  constexpr int PER = 16 / sizeof(KVT);
  constexpr int CPR = DH / PER;
  const KVT* kv = static_cast<const KVT*>(a.kv);
#pragma unroll 1
  for (int i = tid; i < 2 * n * CPR; i += nthr) {
    const int c = i % CPR, r = i / CPR;
    const int kvsel = r >= n, key = kvsel ? r - n : r, pos = t0 + key;
    const int page = max(pg[pos / a.PT - t0 / a.PT], 0);
    const KVT* src = kv + ((((size_t)page * a.L + a.layer) * 2 + kvsel) * a.H + h) * (size_t)a.PT * DH + (size_t)(pos % a.PT) * DH;
    const int cs = kv_swizzled<DH, KVT>() ? (c ^ (pos & 7)) : c;  // the stored piece
    cp_async16((kvsel ? vs : ks) + key * ST + c * PER, src + cs * PER, 16);
  }
}

template <int DH, typename KVT>
__device__ __forceinline__ void attn_load_kv(const AttnArgs& a, int seq, int h, int t0, int lo, int hi, KVT* ks, KVT* vs, int tid,
                                             int nthr) {
  constexpr int PER = 16 / sizeof(KVT);
  constexpr int CPR = DH / PER;
  constexpr int ST = kv_stride<DH, KVT>();
  const int n = max(0, hi - lo);
#pragma unroll 1
  for (int i = tid; i < 2 * n; i += nthr) {
    const int kvsel = i >= n;
    const int key = lo - t0 + (kvsel ? i - n : i);
    const KVT* src = kv_chunk_src<DH, KVT>(a, seq, h, t0 + key, kvsel);
    KVT* dst = (kvsel ? vs : ks) + key * ST;
    const int sw = kv_swizzled<DH, KVT>() ? ((t0 + key) & 7) : 0;  // stored pieces are permuted by position
#pragma unroll
    for (int c = 0; c < CPR; ++c) cp_async16(dst + c * PER, src + (c ^ sw) * PER, 16);
  }
}

// Scores of rows 0..nr-1 against each key: s[r] = sum_c q[r][c] k[c], one
// fmaf chain in c order.  `per` threads share a key (thread `part` takes rows
// part, part + per, ...).  The key is widened 32 columns at a time and the
// running sums live in ps between column blocks (an exact round trip), which
// keeps the loop small for the instruction cache.  ST: row stride of ks.
template <int DH, typename KVT, int ST = kv_stride<DH, KVT>()>
__device__ __forceinline__ void attn_scores(int CH, const float* qs, const KVT* ks, float* ps, const int* lim, int nr, int nk, int tid,
                                            int nthr) {
  constexpr int CB = DH < 32 ? DH : 32;  // columns per block
  const int per = max(1, nthr / CH);
  for (int idx = tid; idx < CH * per; idx += nthr) {
    const int key = idx % CH, part = idx / CH;
    if (key < nk) {
      for (int c0 = 0; c0 < DH; c0 += CB) {
        float kf[CB];
#pragma unroll
        for (int c8 = 0; c8 < CB / 8; ++c8) widen8(ks + key * ST + c0 + c8 * 8, kf + c8 * 8);
#pragma unroll 1
        for (int r = part; r < nr; r += per) {
          const float* q = qs + r * DH + c0;
          float sr = (c0 == 0) ? 0.f : ps[r * CH + key];
#pragma unroll
          for (int c4 = 0; c4 < CB / 4; ++c4) {
            const float4 qv = *reinterpret_cast<const float4*>(q + c4 * 4);
            sr = fmaf(qv.x, kf[c4 * 4 + 0], sr);
            sr = fmaf(qv.y, kf[c4 * 4 + 1], sr);
            sr = fmaf(qv.z, kf[c4 * 4 + 2], sr);
            sr = fmaf(qv.w, kf[c4 * 4 + 3], sr);
          }
          ps[r * CH + key] = sr;
        }
      }
    }
    for (int r = part; r < nr; r += per)
      if (!(key < nk && key < lim[r])) ps[r * CH + key] = -INFINITY;
  }
}

// Four 8x8 b16 matrices from shared memory as one m16n8k16 A fragment (ldmatrix);
// lane L gives the address of row L & 7 of matrix L >> 3 (16 bytes, 16-byte aligned).
// _t: each matrix transposed on the way.
__device__ __forceinline__ uint4 ldsm_x4(const void* p) {
  uint4 r;
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(smem_u32(p))
               : "memory");
  return r;
}
__device__ __forceinline__ uint4 ldsm_x4_t(const void* p) {
  uint4 r;
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(smem_u32(p))
               : "memory");
  return r;
}

// bf16 K/V on the tensor cores.  Scores: S^T (16 keys x 8 rows) = K (16 x 16
// dims, bf16 A operand from smem) . q^T (dims x rows, split into bf16 hi and
// lo B operands), hi then lo per 16-dim step, steps in dim order; one warp
// per (key tile, row group).  Keys past nk or past a row's limit get -inf.
// K rows past nk are never loaded: their scores are discarded.
template <int DH, int ST = kv_stride<DH, __nv_bfloat16>()>
__device__ __forceinline__ void attn_scores_mma(int CH, const float* qs, const __nv_bfloat16* ks, float* ps, const int* lim, int nr,
                                                int nk, int tid, int nthr) {
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3, nw = nthr >> 5;
  const int nkt = CH / 16, nrg = (nr + 7) / 8;
#pragma unroll 1
  for (int item = warp; item < nkt * nrg; item += nw) {
    const int key0 = (item % nkt) * 16, rg = item / nkt;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (key0 < nk) {
      const float* q = qs + min(rg * 8 + g, nr - 1) * DH;  // rows past nr: a live row's values, never stored
      // this lane's row address for ldmatrix: keys key0 + (lane & 7) (+ 8 for matrices 1, 3), dims + 8 for matrices 2, 3
      const int kr = key0 + (lane & 7) + ((lane >> 3) & 1) * 8, kc = (lane >> 4) * 8;
#pragma unroll
      for (int s = 0; s < DH / 16; ++s) {
        const int c = s * 16 + 2 * t;
        const uint4 A = ldsm_x4(ks + kv_at<ST>(kr, s * 16 + kc));  // K[key0 + g | + 8][c, c + 1 | c + 8, c + 9]
        const float2 qa = *reinterpret_cast<const float2*>(q + c), qb = *reinterpret_cast<const float2*>(q + c + 8);
        const XFrag xf = make_xfrag(qa.x, qa.y, qb.x, qb.y);
        mma16816(acc, A, xf.b0h, xf.b1h);
        mma16816(acc, A, xf.b0l, xf.b1l);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = key0 + g + (e >= 2 ? 8 : 0), r = rg * 8 + 2 * t + (e & 1);
      if (r < nr) ps[r * CH + key] = (key < nk && key < lim[r]) ? acc[e] : -INFINITY;
    }
  }
}

// o^T (16 columns x 8 rows) = V^T (16 columns x 16 keys, bf16 A operand
// gathered from smem) . p^T (keys x rows, split into bf16 hi and lo), key
// tiles in order; one warp per (column tile, row group).  V rows from nk up
// to the next multiple of 16 are zero (their p is 0 as well).  Outputs go to
// emit_o(row, column, value); emit_ml(row, m, l) once per row.
template <int DH, int ST, class EmitO, class EmitML>
__device__ __forceinline__ void attn_pv_mma(int CH, const float* ps, const __nv_bfloat16* vs, int nr, int nk, const float* mrow,
                                            const float* lrow, int tid, int nthr, EmitO emit_o, EmitML emit_ml) {
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3, nw = nthr >> 5;
  const int nkt = (nk + 15) / 16, nrg = (nr + 7) / 8;
#pragma unroll 1
  for (int item = warp; item < (DH / 16) * nrg; item += nw) {
    const int c0 = (item % (DH / 16)) * 16, rg = item / (DH / 16);
    const float* p = ps + min(rg * 8 + g, nr - 1) * CH;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    // this lane's row address for ldmatrix.trans: keys (lane & 7) (+ 8 for matrices 2, 3), columns c0 (+ 8 for 1, 3)
    const int vr = (lane & 7) + (lane >> 4) * 8, vc = c0 + ((lane >> 3) & 1) * 8;
#pragma unroll 4
    for (int kt = 0; kt < nkt; ++kt) {
      const int k0 = kt * 16 + 2 * t;
      // V^T fragment: V[k0, k0 + 1 | k0 + 8, k0 + 9][c0 + g | c0 + g + 8]
      const uint4 A = ldsm_x4_t(vs + kv_at<ST>(kt * 16 + vr, vc));
      const float2 pa = *reinterpret_cast<const float2*>(p + k0), pb = *reinterpret_cast<const float2*>(p + k0 + 8);
      const XFrag xf = make_xfrag(pa.x, pa.y, pb.x, pb.y);
      mma16816(acc, A, xf.b0h, xf.b1h);
      mma16816(acc, A, xf.b0l, xf.b1l);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = c0 + g + (e >= 2 ? 8 : 0), r = rg * 8 + 2 * t + (e & 1);
      if (r < nr) {
        emit_o(r, c, acc[e]);
        if (c == 0) emit_ml(r, mrow[r], lrow[r]);
      }
    }
  }
}

// Softmax partial of one chunk of keys for rows 0..nr-1 (per row limit lim):
// m = max score, l = sum exp(s - m), o = sum exp(s - m) v.  On entry qs
// [rows][DH] holds q pre-scaled by 1/sqrt(dh), lim the rows' key limits
// (relative to the chunk), ks/vs the chunk's nk keys (row stride ST; for bf16,
// V rows nk .. next multiple of 16 zeroed), and every thread has passed
// `sync` since they were written.  Outputs through emit_o / emit_ml.
struct NoMark {
  __device__ void operator()(int) const {}
};

// Chunk partial for one or two rows (bf16 K/V), on the CUDA cores: threads 0..127
// take part whatever nthr is (the arithmetic does not depend on the block size).
//   scores: thread t = key t, s_r = fmaf chain over the columns in order (q in
//     fp32, pre-scaled; K widened from bf16).
//   softmax: m_r = max over keys (warp maxima, then the 4 warps in order);
//     p = exp(s - m) (0 for masked keys); l_r = warp sums (butterfly), then the 4
//     warps' sums added in order.
//   PV: thread t = column pair (t mod 32 [+ 32 j]) x key quarter t / 32 (32
//     keys, one fmaf chain in key order); the 4 quarters are added in order.
// Scratch: ps [2][CH] then 16 floats; the K tile, once the scores are taken,
// holds the PV partials [4][2][DH] (CH >= 16 rows of >= DH bf16 hold them).
template <int DH, int ST, class Sync, class EmitO, class EmitML>
__device__ void attn_chunk_small(int CH, const float* qs, float* ps, const __nv_bfloat16* ks, const __nv_bfloat16* vs, float* mrow,
                                 float* lrow, const int* lim, int nr, int nk, int tid, Sync sync, EmitO emit_o, EmitML emit_ml) {
  constexpr int NC = DH / 8;   // 16-byte pieces of a key row
  constexpr int NP = DH / 2;   // column pairs
  constexpr int PPT = (NP + 31) / 32;
  const int warp = tid >> 5, lane = tid & 31;
  float* red = ps + 2 * CH;    // [2 rows][4 warps] maxima, then sums
  const bool act = tid < 128;
  float s0 = -INFINITY, s1 = -INFINITY;
  if (act && tid < nk) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const uint4 w = *reinterpret_cast<const uint4*>(ks + kv_at<ST>(tid, j * 8));  // columns 8j .. 8j + 7
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        const int c = j * 8 + 2 * e;
        a0 = fmaf(qs[c], f.x, a0);
        a0 = fmaf(qs[c + 1], f.y, a0);
        if (nr > 1) {
          a1 = fmaf(qs[DH + c], f.x, a1);
          a1 = fmaf(qs[DH + c + 1], f.y, a1);
        }
      }
    }
    if (tid < lim[0]) s0 = a0;
    if (nr > 1 && tid < lim[1]) s1 = a1;
  }
  // softmax statistics
  float m0 = warp_max(s0), m1 = warp_max(s1);
  if (act && lane == 0) red[warp] = m0, red[4 + warp] = m1;
  sync();
  m0 = fmaxf(fmaxf(fmaxf(red[0], red[1]), red[2]), red[3]);
  m1 = fmaxf(fmaxf(fmaxf(red[4], red[5]), red[6]), red[7]);
  const float p0 = (s0 == -INFINITY) ? 0.f : expf(s0 - m0);
  const float p1 = (s1 == -INFINITY) ? 0.f : expf(s1 - m1);
  if (act && tid < CH) {
    ps[tid] = p0;
    ps[CH + tid] = p1;
  }
  const float l0 = warp_sum(p0), l1 = warp_sum(p1);
  if (act && lane == 0) red[8 + warp] = l0, red[12 + warp] = l1;
  sync();
  if (tid == 0) {
    mrow[0] = m0, lrow[0] = ((red[8] + red[9]) + red[10]) + red[11];
    if (nr > 1) mrow[1] = m1, lrow[1] = ((red[12] + red[13]) + red[14]) + red[15];
  }
  // PV partials of key quarter `warp`, into the K tile (no thread reads K any more)
  float* part = reinterpret_cast<float*>(const_cast<__nv_bfloat16*>(ks));
  const int kq = warp;
  if (act) {
#pragma unroll
    for (int j = 0; j < PPT; ++j) {
      const int cp = lane + 32 * j;
      if (cp < NP) {
        float o00 = 0.f, o01 = 0.f, o10 = 0.f, o11 = 0.f;
        const int k1 = min(kq * 32 + 32, nk);
#pragma unroll 4
        for (int k = kq * 32; k < k1; ++k) {
          const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vs + kv_at<ST>(k, 2 * cp)));
          const float q0 = ps[k], q1 = ps[CH + k];
          o00 = fmaf(q0, v.x, o00);
          o01 = fmaf(q0, v.y, o01);
          if (nr > 1) {
            o10 = fmaf(q1, v.x, o10);
            o11 = fmaf(q1, v.y, o11);
          }
        }
        float* pr = part + (size_t)kq * 2 * DH;  // [quarter][row][DH]
        pr[2 * cp] = o00, pr[2 * cp + 1] = o01;
        pr[DH + 2 * cp] = o10, pr[DH + 2 * cp + 1] = o11;
      }
    }
  }
  sync();
  for (int i = tid; i < nr * DH; i += 128) {
    if (!act) break;
    const int r = i / DH, c = i % DH;
    const float o = ((part[r * DH + c] + part[2 * DH + r * DH + c]) + part[4 * DH + r * DH + c]) + part[6 * DH + r * DH + c];
    emit_o(r, c, o);
  }
  if (tid < nr) emit_ml(tid, mrow[tid], lrow[tid]);
}


template <int DH, typename KVT, int ST, class Sync, class EmitO, class EmitML, class Mark = NoMark>
__device__ void attn_chunk_core(int CH, const float* qs, float* ps, const KVT* ks, const KVT* vs, float* mrow, float* lrow,
                                const int* lim, int nr, int nk, int tid, int nthr, Sync sync, EmitO emit_o, EmitML emit_ml,
                                Mark mark = Mark()) {
  mark(1);
  if constexpr (sizeof(KVT) == 2) {
    if (nr <= 2 && CH <= 128) {  // one or two rows: the CUDA-core path (any block size, the same bits)
      attn_chunk_small<DH, ST>(CH, qs, ps, ks, vs, mrow, lrow, lim, nr, nk, tid, sync, emit_o, emit_ml);
      mark(3);
      return;
    }
  }
  if constexpr (sizeof(KVT) == 2) attn_scores_mma<DH, ST>(CH, qs, ks, ps, lim, nr, nk, tid, nthr);
  else attn_scores<DH, KVT, ST>(CH, qs, ks, ps, lim, nr, nk, tid, nthr);
  sync();
  mark(2);
  const int warp = tid >> 5, lane = tid & 31, nw = nthr >> 5;
#pragma unroll 1
  for (int r = warp; r < nr; r += nw) {
    float m = -INFINITY;
    float l = 0.f;
    if (CH == 128) {  // the usual chunk: a lane's four scores loaded at once, the exps in parallel
      float s[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) s[j] = ps[r * CH + lane + 32 * j];
      m = fmaxf(fmaxf(fmaxf(m, s[0]), s[1]), fmaxf(s[2], s[3]));
      m = warp_max(m);
      float p[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        p[j] = (s[j] == -INFINITY) ? 0.f : expf(s[j] - m);
        ps[r * CH + lane + 32 * j] = p[j];
      }
      l = ((p[0] + p[1]) + p[2]) + p[3];  // 0 + p0 = p0: the same sums as the loop below
    } else {
#pragma unroll 1
      for (int k = lane; k < CH; k += 32) m = fmaxf(m, ps[r * CH + k]);
      m = warp_max(m);
#pragma unroll 1
      for (int k = lane; k < CH; k += 32) {
        const float s = ps[r * CH + k];
        const float p = (s == -INFINITY) ? 0.f : expf(s - m);
        ps[r * CH + k] = p;
        l += p;
      }
    }
    l = warp_sum(l);
    if (lane == 0) {
      mrow[r] = m;
      lrow[r] = l;
    }
  }
  sync();
  mark(3);
  if constexpr (sizeof(KVT) == 2) {
    attn_pv_mma<DH, ST>(CH, ps, vs, nr, nk, mrow, lrow, tid, nthr, emit_o, emit_ml);
    return;
  }
  // o[r][c] = sum_k p[r][k] v[k][c], one fmaf chain in k order per output.
  // A thread owns column c and rows r0, r0 + rs, ... four at a time, so each
  // V element it loads feeds four chains.  (nthr is a multiple of DH.)
  const int c = tid % DH, rs = nthr / DH;
#pragma unroll 1
  for (int r0 = tid / DH; r0 < nr; r0 += 4 * rs) {
    int rr[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) rr[j] = min(r0 + j * rs, nr - 1);  // rows past nr repeat a live one, not stored
    float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int k = 0; k < nk; ++k) {
      float v;
      if constexpr (sizeof(KVT) == 2) v = __bfloat162float(vs[kv_at<ST>(k, c)]);
      else v = vs[kv_at<ST>(k, c)];
#pragma unroll
      for (int j = 0; j < 4; ++j) o[j] = fmaf(ps[rr[j] * CH + k], v, o[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = r0 + j * rs;
      if (r < nr) {
        emit_o(r, c, o[j]);
        if (c == 0) emit_ml(r, mrow[r], lrow[r]);
      }
    }
  }
}

// Softmax partial of one (group, head, chunk) of the per-phase path, in two
// steps: attn_partial_stage loads q and the row limits into smem and zeroes the
// V padding (it may run while the chunk's K/V copies are in flight); after the
// caller's wait and `sync`, attn_partial_run runs attn_chunk_core with the
// partials to a.part_o / a.part_ml.  ROWS: the smem capacity in rows (the
// group's row count must not exceed it).
template <int DH, typename KVT, int ROWS, int ST>
__device__ __forceinline__ bool attn_partial_stage(const AttnArgs& a, int gi, int h, int chunk, float* qs, KVT* vs, int* lim,
                                                   int tid, int nthr) {
  const int row0 = __ldcg(a.rows.g_row0 + gi), nr = __ldcg(a.rows.g_nrows + gi), kmax = __ldcg(a.rows.g_kmax + gi);
  if (nr > ROWS) {  // the host's bound on rows per group was wrong: no write past the smem
    if (tid == 0) set_status(a.status, kErrDevice);
    return false;
  }
  const int t0 = chunk * a.CH;
  const int nk = min(a.CH, kmax - t0);
  for (int i = tid; i < nr * DH; i += nthr) {
    const int r = i / DH, c = i % DH;
    qs[r * DH + c] = __ldcg(a.q + (size_t)(row0 + r) * a.d + h * DH + c) * a.scale;
  }
  if (tid < ROWS) lim[tid] = (tid < nr) ? __ldcg(a.rows.nkeys + row0 + tid) - t0 : 0;
  if constexpr (sizeof(KVT) == 2) {  // zero V rows nk .. next multiple of 16 (read by the last key tile)
    const int pad = ((nk + 15) & ~15) - nk;
    for (int i = tid; i < pad * (DH / 8); i += nthr)
      *reinterpret_cast<uint4*>(vs + (nk + i / (DH / 8)) * ST + (i % (DH / 8)) * 8) = make_uint4(0, 0, 0, 0);
  }
  return true;
}
template <int DH, typename KVT, int ROWS, int ST, class Sync>
__device__ __forceinline__ void attn_partial_run(const AttnArgs& a, int gi, int h, int chunk, const float* qs, float* ps, const KVT* ks,
                                                 const KVT* vs, float* mrow, float* lrow, const int* lim, int tid, int nthr, Sync sync) {
  const int row0 = __ldcg(a.rows.g_row0 + gi), nr = __ldcg(a.rows.g_nrows + gi), kmax = __ldcg(a.rows.g_kmax + gi);
  const int nk = min(a.CH, kmax - chunk * a.CH);
  attn_chunk_core<DH, KVT, ST>(
      a.CH, qs, ps, ks, vs, mrow, lrow, lim, nr, nk, tid, nthr, sync,
      [&](int r, int c, float v) { a.part_o[(((size_t)(row0 + r) * a.H + h) * a.CMAX + chunk) * DH + c] = v; },
      [&](int r, float m, float l) { a.part_ml[((size_t)(row0 + r) * a.H + h) * a.CMAX + chunk] = make_float2(m, l); });
}

// att[h*dh + c] = sum_chunks o_c e^{m_c - m} / sum_chunks l_c e^{m_c - m} for
// one (row, head) by one warp, over nch chunks.  m = largest chunk maximum
// (chunks with l > 0); lane j holds the weight of chunk j of each 32-chunk
// block; l is the warp sum of the lanes' l_c w_c sums; o accumulates the
// chunks in order with the weight broadcast from its lane.  Lane c (and
// c + 32, ...) owns column c.  ml(ch) -> float2 (m, l); ov(ch, col) -> o;
// out(col, value).
template <int DH, class ML, class OV, class Out>
__device__ __forceinline__ void attn_combine(int nch, int lane, ML ml_at, OV o_at, Out out) {
  constexpr int DPL = DH >= 32 ? DH / 32 : 1;  // columns per lane
  float m = -INFINITY;
#pragma unroll 1
  for (int ch = lane; ch < nch; ch += 32) {
    const float2 ml = ml_at(ch);
    if (ml.y > 0.f) m = fmaxf(m, ml.x);
  }
  m = warp_max(m);
  float l = 0.f, o[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) o[i] = 0.f;
  const bool col_ok = lane < DH;
#pragma unroll 1
  for (int cb = 0; cb < nch; cb += 32) {
    float w = 0.f;
    if (cb + lane < nch) {
      const float2 ml = ml_at(cb + lane);
      if (ml.y > 0.f) {
        w = expf(ml.x - m);
        l = fmaf(ml.y, w, l);
      }
    }
    const int nb = min(32, nch - cb);
#pragma unroll 1
    for (int j0 = 0; j0 < nb; j0 += 4) {
      float ov[4][DPL], wj[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        wj[j] = __shfl_sync(0xffffffffu, w, (j0 + j) & 31);
        const int ch = cb + min(j0 + j, nb - 1);
#pragma unroll
        for (int i = 0; i < DPL; ++i) ov[j][i] = col_ok ? o_at(ch, lane + 32 * i) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (j0 + j < nb)
#pragma unroll
          for (int i = 0; i < DPL; ++i) o[i] = fmaf(ov[j][i], wj[j], o[i]);
    }
  }
  l = warp_sum(l);
  if (col_ok)
#pragma unroll
    for (int i = 0; i < DPL; ++i) out(lane + 32 * i, o[i] / l);
}

template <int DH>
__device__ __forceinline__ void attn_combine_row(const AttnArgs& a, int row, int h, int lane) {
  const int nk = __ldcg(a.rows.nkeys + row);
  const int nch = (nk + a.CH - 1) / a.CH;
  const size_t base = ((size_t)row * a.H + h) * a.CMAX;
  attn_combine<DH>(
      nch, lane, [&](int ch) { return __ldcg(a.part_ml + base + ch); },
      [&](int ch, int col) { return __ldcg(a.part_o + (base + ch) * DH + col); },
      [&](int col, float v) { a.att[(size_t)row * a.d + h * DH + col] = v; });
}

// grid (H, chunks, groups); 128 threads.
// grid (H, chunks, groups), 128 threads; ROWS: rows per group at most (smem).
template <int DH, typename KVT, int ROWS>
__global__ void __launch_bounds__(128) k_attn_partial(AttnArgs a) {
  constexpr int ST = kv_stride<DH, KVT>();
  const int gi = blockIdx.z;
  if (gi >= *a.rows.n_groups) return;
  const int kmax = a.rows.g_kmax[gi];
  const int t0 = blockIdx.y * a.CH;
  if (t0 >= kmax) return;
  const int h = blockIdx.x;
  extern __shared__ float4 smem4[];
  float* qs = reinterpret_cast<float*>(smem4);
  float* ps = qs + ROWS * DH;
  KVT* ks = reinterpret_cast<KVT*>(ps + ROWS * a.CH);
  KVT* vs = ks + a.CH * ST;
  __shared__ float mrow[ROWS], lrow[ROWS];
  __shared__ int lim[ROWS];
  __shared__ int pg[16];  // the chunk's KV pages (at most CH / PT + 1 <= 9)
  const int n = min(t0 + a.CH, kmax) - t0;
  const int p0 = t0 / a.PT, np = (t0 + n - 1) / a.PT - p0 + 1;
  if (threadIdx.x < np) {
    const int seq = a.rows.g_seq[gi], pi = p0 + threadIdx.x;
    int page = (pi < a.max_pages) ? a.page_table[seq * a.max_pages + pi] : -1;
    if (page < 0) set_status(a.status, kErrDevice);
    pg[threadIdx.x] = page;
  }
  // q and the row limits load while the page ids do; then every K/V copy goes out at once
  const bool ok = attn_partial_stage<DH, KVT, ROWS, ST>(a, gi, h, blockIdx.y, qs, vs, lim, threadIdx.x, 128);
  __syncthreads();
  attn_load_kv_paged<DH, KVT>(a, pg, h, t0, n, ks, vs, threadIdx.x, 128);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  if (!ok) return;
  attn_partial_run<DH, KVT, ROWS, ST>(a, gi, h, blockIdx.y, qs, ps, ks, vs, mrow, lrow, lim, threadIdx.x, 128,
                                      [] { __syncthreads(); });
}

// grid (rows_max, H), one warp.
template <int DH>
__global__ void __launch_bounds__(32) k_attn_combine(AttnArgs a) {
  const int row = blockIdx.x;
  if (row >= *a.rows.n_rows) return;
  attn_combine_row<DH>(a, row, blockIdx.y, threadIdx.x);
}

// ------------------------------------------------------------------------ byte head statistics
// Over the 256 byte logits of a row (one warp): confidence = largest softmax
// probability, argmax (lowest byte on ties), gap between the two largest
// logits, and the entropy (nats) of the softmax: with e_i = exp(z_i - max),
// S = sum e_i and T = sum e_i (z_i - max), H = ln S - T / S.
__device__ __forceinline__ void head_stats_row(const float* z, int lane, float& conf, int& pred, float& gap, float& ent) {
  float v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = __ldcg(z + lane + 32 * j);
  float b1 = -INFINITY, b2 = -INFINITY;
  int i1 = 1 << 30;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int idx = lane + 32 * j;
    if (v[j] > b1) {
      b2 = b1;
      b1 = v[j];
      i1 = idx;
    } else {
      b2 = fmaxf(b2, v[j]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ob1 = __shfl_xor_sync(0xffffffffu, b1, o);
    const float ob2 = __shfl_xor_sync(0xffffffffu, b2, o);
    const int oi1 = __shfl_xor_sync(0xffffffffu, i1, o);
    if (ob1 > b1 || (ob1 == b1 && oi1 < i1)) {
      b2 = fmaxf(b1, ob2);
      b1 = ob1;
      i1 = oi1;
    } else {
      b2 = fmaxf(b2, ob1);
    }
  }
  float s = 0.f, tz = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float e = expf(v[j] - b1);
    s += e;
    tz = fmaf(e, v[j] - b1, tz);
  }
  s = warp_sum(s);
  tz = warp_sum(tz);
  conf = 1.0f / s;
  pred = i1;
  gap = b1 - b2;
  ent = logf(s) - tz / s;
}

__global__ void k_head_stats(const float* __restrict__ logits, const int* n_rows, float* conf, int* pred, float* gap, float* ent) {
  const int n = *n_rows;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int r = warp; r < n; r += nw) {
    float c, g, e;
    int p;
    head_stats_row(logits + (size_t)r * 256, lane, c, p, g, e);
    if (lane == 0) {
      conf[r] = c;
      pred[r] = p;
      gap[r] = g;
      ent[r] = e;
    }
  }
}

// ------------------------------------------------------------------------ planning
// Builds the rows of a pass (one CTA, nthr threads; sh: 3*(kMaxCallBatch+1)
// ints of shared memory).  Sequences' rows are contiguous, so each attention
// group (<= 32 rows) belongs to one sequence.  row_off / lat_off may be NULL
// (no pending rows / latents).
template <class Sync>
__device__ void plan_rows(const PlanArgs& p, int B, const int* row_off, const int* lat_off, SeqDev sd, RowsDev rd, int tid,
                          int nthr, int* sh, Sync sync) {
  int* cnt = sh;
  int* gcnt = sh + (kMaxCallBatch + 1);
  int* npend = sh + 2 * (kMaxCallBatch + 1);
  if (tid == 0) {
    int off = 0, goff = 0;
    for (int s = 0; s < B; ++s) {
      const int np = row_off ? row_off[s + 1] - row_off[s] : 0;
      int n = 0;
      if (p.mode == PL_PREFILL) {
        const int lo = max(row_off[s], p.r0), hi = min(row_off[s + 1], p.r1);
        n = max(0, hi - lo);
      } else if (p.mode == PL_FIRST) {
        n = np + p.k;
      } else if (p.mode == PL_BLOCK) {
        n = sd.active[s] ? p.k : 0;
      } else if (p.mode == PL_ARDRAFT) {
        n = 1;
      } else {
        n = p.k;
      }
      npend[s] = np;
      cnt[s] = off;
      gcnt[s] = goff;
      off += n;
      goff += (n + kAttnRows - 1) / kAttnRows;
    }
    cnt[B] = off;
    gcnt[B] = goff;
    *rd.n_rows = off;
    *rd.n_groups = goff;
  }
  sync();
  const int n_rows = cnt[B];
  for (int r = tid; r < n_rows; r += nthr) {
    int lo = 0, hi = B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (cnt[mid] <= r) lo = mid;
      else hi = mid;
    }
    const int s = lo, i = r - cnt[s];
    int pos, lat, byte, nkeys, blk_i = -1;
    const int kvl = sd.kv_len[s];
    const int nl = sd.n_lat[s];
    if (p.mode == PL_PREFILL) {
      const int src = max(row_off[s], p.r0) + i;
      pos = sd.kv_base[s] + (src - row_off[s]);
      byte = p.pend_bytes[src];
      lat = p.pend_lat[src];
      nkeys = pos + 1;
    } else if (p.mode == PL_FIRST) {
      const int np = npend[s];
      if (i < np) {
        const int src = row_off[s] + i;
        pos = kvl + i;
        byte = p.pend_bytes[src];
        lat = p.pend_lat[src];
        nkeys = pos + 1;
        if (i == np - 1) sd.last_row[s] = r;
      } else {
        blk_i = i - np;
        pos = kvl + i;
        byte = p.mask_id;
        lat = nl - 1;
        nkeys = kvl + np + p.k;
      }
    } else if (p.mode == PL_BLOCK) {
      blk_i = i;
      pos = kvl + i;
      byte = sd.masked[s * kMaxBlock + i] ? p.mask_id : sd.blk[s * kMaxBlock + i];
      lat = nl - 1;
      nkeys = kvl + p.k;
    } else if (p.mode == PL_ARDRAFT) {
      blk_i = 0;
      pos = kvl + p.step - 1;
      byte = sd.blk[s * kMaxBlock + p.step - 1];
      lat = nl - 1;
      nkeys = pos + 1;
    } else {  // PL_VERIFY
      blk_i = i;
      pos = kvl + i;
      byte = sd.blk[s * kMaxBlock + i];
      lat = p.vlat[s * p.k + i];
      nkeys = pos + 1;
    }
    const int lat_cap = nl + ((p.mode == PL_VERIFY && lat_off) ? (lat_off[s + 1] - lat_off[s]) : 0);
    if (pos < 0 || pos >= p.max_ctx || lat < 0 || lat >= lat_cap || lat >= p.max_lat || byte < 0 || byte > p.mask_id) {
      set_status(sd.status, kErrDevice);
      pos = min(max(pos, 0), p.max_ctx - 1);
      lat = 0;
      byte = 0;
      nkeys = min(max(nkeys, 1), pos + 1);
    }
    rd.seq[r] = s;
    rd.pos[r] = pos;
    rd.lat[r] = lat;
    rd.byte[r] = byte;
    rd.nkeys[r] = nkeys;
    if (blk_i >= 0) sd.blk_row[s * kMaxBlock + blk_i] = r;
  }
  for (int gi = tid; gi < gcnt[B]; gi += nthr) {
    int lo = 0, hi = B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (gcnt[mid] <= gi) lo = mid;
      else hi = mid;
    }
    const int s = lo, j = gi - gcnt[s];
    const int r0 = cnt[s] + kAttnRows * j;
    rd.g_seq[gi] = s;
    rd.g_row0[gi] = r0;
    rd.g_nrows[gi] = min(kAttnRows, cnt[s + 1] - r0);
  }
  sync();
  for (int gi = tid; gi < gcnt[B]; gi += nthr) {
    int km = 0;
    for (int r = rd.g_row0[gi]; r < rd.g_row0[gi] + rd.g_nrows[gi]; ++r) km = max(km, rd.nkeys[r]);
    rd.g_kmax[gi] = km;
    rd.g_fresh[gi] = rd.pos[cnt[rd.g_seq[gi]]];  // positions this pass writes start at the sequence's first row
  }
  sync();
  if (tid == 0) {
    if (p.mode == PL_FIRST) {
      for (int s = 0; s < B; ++s) {
        if (npend[s] == 0) sd.last_row[s] = -1;
        sd.kv_len[s] += npend[s];
        if (p.k > 0) {
          sd.active[s] = 1;
          sd.steps[s] = 0;
          for (int i = 0; i < p.k; ++i) sd.masked[s * kMaxBlock + i] = 1;
        }
      }
    }
    if (n_rows > 0) {
      unsigned long long kvk = 0;  // algorithmic K/V bytes: each sequence's keys read once per layer
      for (int gi = 0; gi < gcnt[B]; ++gi) {
        if (gi == 0 || rd.g_seq[gi - 1] != rd.g_seq[gi]) {
          int km = 0;
          for (int gj = gi; gj < gcnt[B] && rd.g_seq[gj] == rd.g_seq[gi]; ++gj) km = max(km, rd.g_kmax[gj]);
          kvk += km;
        }
      }
      if (p.mode == PL_PREFILL) {
        sd.counters[2] += n_rows;
        sd.counters[7] += kvk * p.kv_bytes_per_key;
      } else {
        sd.counters[0] += 1;
        sd.counters[5] += p.weight_bytes_per_pass;
        sd.counters[6] += kvk * p.kv_bytes_per_key;
      }
      sd.counters[1] += n_rows;
    }
  }
  sync();
}

__global__ void __launch_bounds__(256) k_plan(PlanArgs p, CallDesc cd, SeqDev sd, RowsDev rd) {
  __shared__ int sh[3 * (kMaxCallBatch + 1)];
  plan_rows(p, cd.batch, cd.row_off, cd.lat_off, sd, rd, threadIdx.x, blockDim.x, sh, [] { __syncthreads(); });
}

// Latent rows: new latent j of sequence s goes to slot n_lat[s] + (j - lat_off[s]).
__global__ void k_lat_plan(CallDesc cd, SeqDev sd, int* lat_seq, int* lat_slot, int* n_lat_rows, int r0, int r1, int commit,
                           int max_lat) {
  const int B = cd.batch;
  for (int j = r0 + threadIdx.x; j < r1; j += blockDim.x) {
    int lo = 0, hi = B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (cd.lat_off[mid] <= j) lo = mid;
      else hi = mid;
    }
    const int slot = sd.n_lat[lo] + (j - cd.lat_off[lo]);
    lat_seq[j - r0] = lo;
    lat_slot[j - r0] = min(slot, max_lat - 1);
    if (slot >= max_lat) set_status(sd.status, kErrDevice);
  }
  if (threadIdx.x == 0) *n_lat_rows = r1 - r0;
  __syncthreads();
  if (commit && threadIdx.x == 0 && r1 == cd.lat_off[B]) {
    for (int s = 0; s < B; ++s) sd.n_lat[s] += cd.lat_off[s + 1] - cd.lat_off[s];
    sd.counters[3] += cd.lat_off[B];
  }
}

// ------------------------------------------------------------------------ bookkeeping (one warp per sequence)
// Block unmasking ("블록 언마스킹 전략"), one warp per sequence, lane = block
// position.  Confidence rule (ent == NULL): every masked position with
// conf >= alpha is committed; if none, the most confident one (lowest position
// on ties).  EB sampling (ent != NULL, bound gamma = alpha): masked positions
// ranked by entropy (position breaks ties), running sums of entropy taken in
// rank order in fp32, every position whose running sum is <= gamma is
// committed, and at least the first.  Returns whether masked positions remain.
// newly (optional): the lanes committed by this pass; with greedy_bytes false the
// caller writes their bytes (sampling).
__device__ __forceinline__ bool unmask_seq(SeqDev sd, int s, int batch, int k, float alpha, int step, const float* conf,
                                           const int* pred, const float* logits, float* out_logits, int lane,
                                           const float* ent = nullptr, unsigned* newly = nullptr, bool greedy_bytes = true) {
  if (step == 0 && lane == 0) {
    const int lr = sd.last_row[s];
    if (lr >= 0) sd.y_last[s] = __ldcg(pred + lr);
  }
  const bool in = lane < k;
  const int row = in ? sd.blk_row[s * kMaxBlock + lane] : 0;
  const bool m = in && sd.masked[s * kMaxBlock + lane];
  const float c = m ? __ldcg(conf + row) : -1.0f;
  const bool over = !ent && m && (c >= alpha);
  const unsigned any_over = __ballot_sync(0xffffffffu, over);
  bool commit = over;
  if (ent) {
    const float e = m ? __ldcg(ent + row) : INFINITY;
    const unsigned mm = __ballot_sync(0xffffffffu, m);
    int rank = 0;
    for (int j = 0; j < 32; ++j) {
      const float ej = __shfl_sync(0xffffffffu, e, j);
      if (((mm >> j) & 1u) && (ej < e || (ej == e && j < lane))) ++rank;
    }
    float run = 0.f, cum = 0.f;
    const int nm = __popc(mm);
    for (int r = 0; r < nm; ++r) {
      const int src = __ffs(__ballot_sync(0xffffffffu, m && rank == r)) - 1;
      run += __shfl_sync(0xffffffffu, e, src);
      if (m && rank == r) cum = run;
    }
    commit = m && (cum <= alpha || rank == 0);
  } else if (!any_over) {
    float best = c;
    int bi = m ? lane : 1 << 30;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob > best || (ob == best && oi < bi)) {
        best = ob;
        bi = oi;
      }
    }
    commit = m && lane == bi;
  }
  if (commit) {
    if (greedy_bytes) sd.blk[s * kMaxBlock + lane] = (unsigned char)__ldcg(pred + row);
    sd.masked[s * kMaxBlock + lane] = 0;
  }
  if (newly) *newly = __ballot_sync(0xffffffffu, commit);
  const unsigned left = __ballot_sync(0xffffffffu, m && !commit);
  if (out_logits && in) {
    float* dst = out_logits + (((size_t)step * batch + s) * k + lane) * 256;
    const float* src = logits + (size_t)row * 256;
    for (int j = 0; j < 256; ++j) dst[j] = __ldcg(src + j);
  }
  if (lane == 0) {
    sd.steps[s] += 1;
    sd.active[s] = left != 0;
  }
  return left != 0;
}

__global__ void k_unmask(SeqDev sd, int batch, int k, float alpha, int step, const float* conf, const int* pred,
                         const float* logits, float* out_logits, const float* ent) {
  const int s = blockIdx.x, lane = threadIdx.x;
  if (s >= batch || !sd.active[s]) return;
  unmask_seq(sd, s, batch, k, alpha, step, conf, pred, logits, out_logits, lane, ent);
}

// AR draft: the argmax of this pass's row becomes draft byte `step`.
__device__ __forceinline__ void draft_ar_seq(SeqDev sd, int s, int batch, int step, const int* pred, const float* logits,
                                             float* out_logits, int lane) {
  const int row = (step == 0) ? sd.last_row[s] : sd.blk_row[s * kMaxBlock];
  if (lane == 0) {
    const int b = __ldcg(pred + row);
    sd.blk[s * kMaxBlock + step] = (unsigned char)b;
    if (step == 0) sd.y_last[s] = b;
  }
  if (out_logits) {
    float* dst = out_logits + ((size_t)step * batch + s) * 256;
    for (int j = lane; j < 256; j += 32) dst[j] = __ldcg(logits + (size_t)row * 256 + j);
  }
}

__global__ void k_draft_ar(SeqDev sd, int batch, int step, const int* pred, const float* logits, float* out_logits) {
  const int s = blockIdx.x;
  if (s < batch) draft_ar_seq(sd, s, batch, step, pred, logits, out_logits, threadIdx.x);
}

// Greedy verification ("BLT-S와 BLT-DV"): with y_slot[i] the greedy byte for
// draft slot i (slot 0: prediction of the last committed row; slot i > 0: of
// draft row i-1), accept while draft[i] == y_slot[i]; the next byte is
// y_slot[a], or the prediction of the last draft row when all k match.
__device__ __forceinline__ void accept_seq(SeqDev sd, int s, int k, const int* pred, const int* vlat, const float* logits,
                                           int* out_acc, unsigned char* out_next, float* out_logits, int lane) {
  const bool in = lane < k;
  const int row = in ? sd.blk_row[s * kMaxBlock + lane] : 0;
  const int y_self = in ? __ldcg(pred + row) : -1;
  const int y_up = __shfl_up_sync(0xffffffffu, y_self, 1);
  const int y_slot = (lane == 0) ? sd.y_last[s] : y_up;
  const bool match = in && (int)sd.blk[s * kMaxBlock + lane] == y_slot;
  const unsigned mm = __ballot_sync(0xffffffffu, !match);
  const int a = (mm == 0u) ? k : min(__ffs(mm) - 1, k);
  const int y_a = __shfl_sync(0xffffffffu, y_slot, a & 31);
  const int y_k = __shfl_sync(0xffffffffu, y_self, (k - 1) & 31);
  if (out_logits && in) {
    float* dst = out_logits + ((size_t)s * k + lane) * 256;
    for (int j = 0; j < 256; ++j) dst[j] = __ldcg(logits + (size_t)row * 256 + j);
  }
  if (lane == 0) {
    const int nxt = (a == k) ? y_k : y_a;
    out_acc[s] = a;
    out_next[s] = (unsigned char)nxt;
    sd.kv_len[s] += a;
    if (a >= 1) sd.n_lat[s] = max(sd.n_lat[s], vlat[s * k + a - 1] + 1);
  }
}

__global__ void k_accept(SeqDev sd, int batch, int k, const int* pred, const int* vlat, const float* logits, int* out_acc,
                         unsigned char* out_next, float* out_logits) {
  const int s = blockIdx.x;
  if (s < batch) accept_seq(sd, s, k, pred, vlat, logits, out_acc, out_next, out_logits, threadIdx.x);
}

// After a block loop: copy blocks out; masked positions left -> STEP_LIMIT.
__global__ void k_finish_block(SeqDev sd, int batch, int k, unsigned char* out_block, int* out_steps) {
  const int s = blockIdx.x, lane = threadIdx.x;
  if (s >= batch) return;
  if (lane < k) out_block[s * k + lane] = sd.blk[s * kMaxBlock + lane];
  if (lane == 0) {
    if (out_steps) out_steps[s] = sd.steps[s];
    if (sd.active[s]) set_status(sd.status, kErrStepLimit);
  }
}

__global__ void k_copy_draft(SeqDev sd, int batch, int k, unsigned char* out) {
  const int s = blockIdx.x, lane = threadIdx.x;
  if (s < batch && lane < k) out[s * k + lane] = sd.blk[s * kMaxBlock + lane];
}

// Page table updates (entries by value).
struct PageUpd {
  int n;
  int idx[64];
  int page[64];
};
__global__ void k_page_update(int* pt, PageUpd u) {
  const int i = threadIdx.x;
  if (i < u.n) pt[u.idx[i]] = u.page[i];
}

// Shrink per-sequence lengths (rewind).
__global__ void k_rewind(SeqDev sd, CallDesc cd) {
  const int s = threadIdx.x;
  if (s < cd.batch) {
    if (cd.row_off[s] >= 0) sd.kv_len[s] = min(sd.kv_len[s], cd.row_off[s]);
    if (cd.lat_off[s] >= 0) sd.n_lat[s] = min(sd.n_lat[s], cd.lat_off[s]);
  }
}

}  // namespace bltdec
