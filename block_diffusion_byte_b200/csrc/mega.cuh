// Persistent decoder-pass kernel: every pass of one C-ABI call (the confidence
// unmasking loop of BLT-D, the k passes of a BLT-S draft, the BLT-DV draft
// loop, or the verification pass) in one cooperative launch, one CTA per SM.
//
// Warp roles: warps 0..7 consume (tensor-core GEMV, attention, bookkeeping),
// warp 8 produces: it streams this CTA's weight pieces and the cached K/V
// pages of its attention items, in the order the consumers use them, through
// a ring of 32 KB shared-memory slots with 1-D bulk copies (L2 evict-first for
// weights).  The producer runs ahead of the consumers across phase boundaries
// (weights do not depend on activations), so HBM keeps streaming while the
// consumers wait for their inputs.
//
// Hand-offs between CTAs use self-validating words: every activation value
// is written as one 64-bit word (epoch << 32 | fp32 bits) with a relaxed
// store, and a consumer polls the words it needs until each carries the
// expected epoch.  A hand-off costs one L2 round trip after the data lands:
// no fence, no flag, no second load.  Epochs are unique per (call, pass,
// layer, stage), so a stale word is never mistaken for a fresh one; a buffer
// is rewritten only after every reader of its previous contents has finished
// (each rewrite depends, through the pass's all-to-all data flow, on outputs
// those readers produced after reading).
//
// Work per layer (G CTAs):
//   QKV   3d/16 units of 16 output rows, unit u on CTA u mod G
//   ATT   items (sequence group, head, 128-key chunk), item i on CTA i mod G;
//         the CTA of chunk 0 combines the head's chunks
//   O     d/16 units, W13 2F/16 units (continuing the round robin)
//   W2    K cut into segments of 1024 columns; segment q has its own G/nseg
//         CTAs; the CTA of the last segment of a unit sums the segments in
//         order and applies the residual.
// The arithmetic of every unit, chunk, combine and bookkeeping step is the
// canonical order of kernels.cuh, so this path and the per-phase kernels give
// bit-identical results.  Every wait is bounded: a wait that runs out sets
// the abort word and the device status (BLT_ERR_DEVICE), and all CTAs leave.
#pragma once

#include <type_traits>

#include "kernels.cuh"

namespace bltdec {

typedef unsigned long long u64;

constexpr int kMegaConsumers = 8;
// Three warpgroups: two of consumers, and one holding the producer warp (its three other
// warps leave at once).  Launched at 168 registers a thread (65536 / 384), the producer's
// warpgroup gives registers back and the consumers take them (setmaxnreg):
// 128 * 56 + 256 * 224 = 384 * 168.
constexpr int kMegaThreads = 12 * 32;
constexpr int kProducerRegs = 64;
constexpr int kConsumerRegs = 216;
static_assert(128 * kProducerRegs + 256 * kConsumerRegs <= kMegaThreads * 168, "register split exceeds the launch's registers");
constexpr int kSlotBytes = 32 * 1024;
constexpr int kRingSlots = 5;
constexpr int kMegaMaxNG = 2;                  // <= 16 rows per pass
constexpr int kMegaRows = 8 * kMegaMaxNG;
constexpr int kMaxPieces = 4;                  // GEMV pieces of one phase reduced together
constexpr int kSegSteps = kSegCols / 16;       // k-steps per canonical K segment

enum MegaMode : int { MM_DIFFUSE = 0, MM_DRAFT_AR = 1, MM_VERIFY = 2 };
// Stage of an exchange word (part of its epoch).
enum Stage : int { ST_QKV = 0, ST_PART = 1, ST_ATT = 2, ST_HO = 3, ST_ACT = 4, ST_W2P = 5, ST_HW = 6, ST_LOGIT = 7 };
enum PhaseKind : int { PH_QKV = 0, PH_O = 1, PH_W13 = 2, PH_W2 = 3, PH_HEAD = 4 };

struct LayerW {
  const uint4* qkv;
  const uint4* o;
  const uint4* w13;
  const uint4* w2;
  const float* attn_norm;
  const float* ffn_norm;
};

struct MegaArgs {
  const LayerW* layers;  // device [L]
  const uint4* whead;
  const float* final_norm;
  int L, d, H, dh, F, planes;
  float eps;
  GemmArgs ga;  // embedding, latent cache, KV pool, page table, rotary tables, shapes
  AttnArgs aa;  // chunk size, scale
  RowsDev rows;
  SeqDev sd;
  // exchange buffers (64-bit words: epoch << 32 | fp32 bits)
  u64* x_h;      // [rows][d] residual stream
  u64* x_q;      // [rows][d] queries (RoPE applied)
  u64* x_k;      // [rows][d] keys of this pass's rows (RoPE applied, rounded like the cache)
  u64* x_v;      // [rows][d] values of this pass's rows (rounded like the cache)
  u64* x_part;   // [rows][H][CMAX][2 + dh] chunk partials (m, l, o)
  u64* x_att;    // [rows][d] attention output
  u64* x_act;    // [rows][F] SwiGLU activations
  u64* x_w2p;    // [nseg - 1][rows][d] W2 segment sums
  u64* x_logit;  // [rows][256]
  int CMAX;
  float* logits;  // [rows][256] plain copy for the bookkeeping
  float* conf;
  float* ent;
  float* gap;
  int* pred;
  int eb;               // block unmasking by EB sampling (bound alpha) instead of confidence
  unsigned* flags;      // [0] decision epoch, [1] pass-end arrivals (zeroed before the launch)
  unsigned* dec_val;    // continue word written with the decision
  unsigned epoch0;
  int* abort;
  unsigned long long wait_ns;  // wall time after which a wait gives up
  unsigned spin_ns0, spin_ns1;  // sleep between polls: the first 32 polls of a wait, then the rest
  int stall_test;       // test only: unit 0 of the first O phase never publishes (a wait must run out)
  unsigned long long* trace;
  int mode, batch, k, max_passes;
  float alpha;
  const int* vlat;
  float* out_logits;
  int* out_acc;
  unsigned char* out_next;
  PlanArgs plan;  // template for the device-side plans of passes >= 2
};

// ---------------------------------------------------------------------------- primitives
__device__ __forceinline__ void tma_1d(void* dst, const void* src, unsigned bytes, uint64_t* b, uint64_t pol) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;\n" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(b)), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void tma_1d_plain(void* dst, const void* src, unsigned bytes, uint64_t* b) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(b))
               : "memory");
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }
// Barrier of the 256 consumer threads that also ANDs a flag across them: every
// control decision after a wait is taken the same way by all consumers.
__device__ __forceinline__ bool consumer_and(bool v) {
  unsigned r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, 256, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((unsigned)v)
      : "memory");
  return r != 0;
}
// generic-proxy writes of this CTA's shared memory become visible to later bulk copies into it
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
// global data written through the generic proxy, read next by bulk copies
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;\n" ::: "memory"); }

// exchange words
__device__ __forceinline__ u64 xw_pack(float v, unsigned e) { return ((u64)e << 32) | (u64)__float_as_uint(v); }
__device__ __forceinline__ bool xw_ok(u64 w, unsigned e) { return (unsigned)(w >> 32) == e; }
__device__ __forceinline__ float xw_val(u64 w) { return __uint_as_float((unsigned)(w & 0xFFFFFFFFull)); }
__device__ __forceinline__ void xw_st(u64* p, float v, unsigned e) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;\n" ::"l"(p), "l"(xw_pack(v, e)) : "memory");
}
__device__ __forceinline__ u64 xw_ld(const u64* p) {
  u64 w;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];\n" : "=l"(w) : "l"(p) : "memory");
  return w;
}
__device__ __forceinline__ void xw_ld2(const u64* p, u64& a, u64& b) {  // p 16-byte aligned; each word read atomically
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];\n" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}

__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// State of one bounded wait: polls so far and when the first one failed.
struct Spin {
  unsigned n = 0;
  unsigned long long t0 = 0;
};
// One step of a bounded wait: back off, count, watch the abort word and the
// clock.  A wait gives up (abort word + BLT_ERR_DEVICE) after m.wait_ns of
// wall time.  False: give up.
__device__ __forceinline__ bool spin_step(const MegaArgs& m, Spin& sp) {
  __nanosleep(sp.n < 32 ? m.spin_ns0 : m.spin_ns1);
  if (sp.n++ == 0) sp.t0 = gtimer();
  if ((sp.n & 31) == 0) {
    if (*(volatile int*)m.abort) return false;
    if (gtimer() - sp.t0 > m.wait_ns) {
      atomicExch(m.abort, 1);
      set_status(m.sd.status, kErrDevice);
      return false;
    }
  }
  return true;
}

// Poll one word until it carries epoch e.
__device__ __forceinline__ bool xw_wait(const MegaArgs& m, const u64* p, unsigned e, float& v) {
  Spin spins;
  while (true) {
    const u64 w = xw_ld(p);
    if (xw_ok(w, e)) {
      v = xw_val(w);
      return true;
    }
    if (!spin_step(m, spins)) return false;
  }
}
// Poll the words idx = tid + 256 i (i < N, idx < n) until each carries epoch
// e; at(idx) is a word's address, put(idx, value) takes its value.  Every load
// of a round is in flight at once; a round re-reads only the words not ready.
template <int N, class At, class Put>
__device__ __forceinline__ bool poll_words(const MegaArgs& m, int n, unsigned e, int tid, At at, Put put) {
  unsigned pending = 0;
#pragma unroll
  for (int i = 0; i < N; ++i)
    if (tid + 256 * i < n) pending |= 1u << i;
  Spin spins;
  if (pending) {  // wait on one word first: a waiting thread issues one load per round, not N
    const int i0 = __ffs(pending) - 1;
    const u64* p0 = at(tid + 256 * i0);
    while (!xw_ok(xw_ld(p0), e))
      if (!spin_step(m, spins)) return false;
  }
  while (pending) {
    u64 w[N];
#pragma unroll
    for (int i = 0; i < N; ++i)
      if ((pending >> i) & 1u) w[i] = xw_ld(at(tid + 256 * i));
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (((pending >> i) & 1u) && xw_ok(w[i], e)) {
        put(tid + 256 * i, xw_val(w[i]));
        pending &= ~(1u << i);
      }
    if (pending && !spin_step(m, spins)) return false;
  }
  return true;
}

// poll_words for pairs of adjacent words (at(i) 16-byte aligned): one 16-byte
// load per pair; put(i, v0, v1) once both words carry epoch e.
template <int N, class At, class Put>
__device__ __forceinline__ bool poll_pairs(const MegaArgs& m, int n, unsigned e, int tid, At at, Put put) {
  unsigned pending = 0;
#pragma unroll
  for (int i = 0; i < N; ++i)
    if (tid + 256 * i < n) pending |= 1u << i;
  Spin spins;
  if (pending) {  // wait on one pair first
    const int i0 = __ffs(pending) - 1;
    const u64* p0 = at(tid + 256 * i0);
    while (true) {
      u64 a, b;
      xw_ld2(p0, a, b);
      if (xw_ok(a, e) && xw_ok(b, e)) break;
      if (!spin_step(m, spins)) return false;
    }
  }
  while (pending) {
    u64 w0[N], w1[N];
#pragma unroll
    for (int i = 0; i < N; ++i)
      if ((pending >> i) & 1u) xw_ld2(at(tid + 256 * i), w0[i], w1[i]);
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (((pending >> i) & 1u) && xw_ok(w0[i], e) && xw_ok(w1[i], e)) {
        put(tid + 256 * i, xw_val(w0[i]), xw_val(w1[i]));
        pending &= ~(1u << i);
      }
    if (pending && !spin_step(m, spins)) return false;
  }
  return true;
}

__device__ __forceinline__ bool wait_mbar(const MegaArgs& m, uint64_t* b, unsigned parity) {
  unsigned n = 0;
  unsigned long long t0 = 0;
  while (!mbar_try(b, parity)) {
    if (n++ == 0) t0 = gtimer();
    if ((n & 255) == 0) {
      if (*(volatile int*)m.abort) return false;
      if (gtimer() - t0 > m.wait_ns) {
        atomicExch(m.abort, 1);
        set_status(m.sd.status, kErrDevice);
        return false;
      }
    }
  }
  return true;
}
__device__ __forceinline__ bool wait_flag(const MegaArgs& m, const unsigned* f, unsigned target, bool eq) {
  Spin spins;
  while (true) {
    const unsigned v = ld_acquire(f);
    if (eq ? v == target : (int)(v - target) >= 0) return true;
    if (!spin_step(m, spins)) return false;
  }
}

__device__ __forceinline__ unsigned epoch(const MegaArgs& m, int pass, int layer, int stage) {
  return m.epoch0 + 1u + (((unsigned)pass * (unsigned)(m.L + 1) + (unsigned)layer) << 3) + (unsigned)stage;
}

// Device-side timestamps (debug): compiled in only with -DBLTDEC_MEGA_TRACE.
constexpr int kTraceEvents = 1024;
__shared__ int s_trace_n;
__device__ __forceinline__ void trace_mark(const MegaArgs& m, int pass, int code) {
#ifdef BLTDEC_MEGA_TRACE
  if (m.trace && pass == 0 && threadIdx.x == 0) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    const int i = s_trace_n++;
    if (i < kTraceEvents) m.trace[(size_t)blockIdx.x * kTraceEvents + i] = ((unsigned long long)code << 48) | (t & 0xFFFFFFFFFFFFull);
  }
#else
  (void)m;
  (void)pass;
  (void)code;
#endif
}
enum TraceCode : int {
  TR_PASS = 1, TR_PH = 2, TR_IN = 3, TR_MMA = 4, TR_DONE = 5, TR_ATT = 6, TR_ATT_DONE = 7, TR_COMB = 8, TR_BOOK = 9,
  TR_SENT = 10, TR_GATH = 11, TR_PRE = 12, TR_ISLOT = 13, TR_IPOLL = 14, TR_ICORE = 15, TR_CBEG = 16,
  TR_CROW = 17, TR_CML = 18, TR_CSUB = 19, TR_ISTAGE = 20, TR_MW = 21
};

// ---------------------------------------------------------------------------- schedule
// Which units (pieces) of a phase a CTA owns: first, first + step, ... (count).
struct Assign {
  int first, step, count;
};
__device__ __forceinline__ Assign rr_assign(int units, int off, int cta, int G) {
  Assign a;
  a.first = ((cta - off) % G + G) % G;
  a.step = G;
  a.count = a.first < units ? (units - a.first + G - 1) / G : 0;
  return a;
}
struct Phase {
  int kind, layer;
  const uint4* w;
  int units;      // output units of 16 rows
  int ksteps;     // K / 16 of the whole matrix
  int seg;        // K segment of this CTA's pieces
  int seg_steps;  // k-steps per piece
  Assign a;
};
__device__ __forceinline__ int n_w2_segments(const MegaArgs& m) { return m.F > kSegCols ? m.F / kSegCols : 1; }

// Phase `kind` of layer `layer` for this CTA (kind PH_HEAD: layer ignored).
__device__ __forceinline__ Phase phase_of(const MegaArgs& m, int kind, int layer, int cta, int G) {
  Phase p;
  p.kind = kind;
  p.layer = layer;
  p.seg = 0;
  const int d = m.d, F = m.F;
  if (kind == PH_HEAD) {
    p.w = m.whead, p.units = 256 / 16, p.ksteps = d / 16;
    p.a = rr_assign(p.units, (4 * d / 16 + 2 * F / 16) % G, cta, G);
  } else {
    const LayerW& lw = m.layers[layer];
    if (kind == PH_QKV) {
      p.w = lw.qkv, p.units = 3 * d / 16, p.ksteps = d / 16;
      p.a = rr_assign(p.units, 0, cta, G);
    } else if (kind == PH_O) {
      p.w = lw.o, p.units = d / 16, p.ksteps = d / 16;
      p.a = rr_assign(p.units, (3 * d / 16) % G, cta, G);
    } else if (kind == PH_W13) {
      p.w = lw.w13, p.units = 2 * F / 16, p.ksteps = d / 16;
      p.a = rr_assign(p.units, (4 * d / 16) % G, cta, G);
    } else {
      p.w = lw.w2, p.units = d / 16, p.ksteps = F / 16;
      const int nseg = n_w2_segments(m), cps = G / nseg;
      const int q = cta / cps;
      p.seg = q;
      if (q < nseg) {
        p.a.first = cta % cps;
        p.a.step = cps;
        p.a.count = p.a.first < p.units ? (p.units - p.a.first + cps - 1) / cps : 0;
      } else {
        p.a.first = 0, p.a.step = 1, p.a.count = 0;
      }
    }
  }
  p.seg_steps = min(p.ksteps, kSegSteps);
  return p;
}
template <int PL>
__device__ __forceinline__ int tiles_per_slot() {
  return kSlotBytes / (512 * PL);
}
template <int PL>
__device__ __forceinline__ int piece_slots(int tiles) {
  return (tiles + tiles_per_slot<PL>() - 1) / tiles_per_slot<PL>();
}

// Attention items of a pass: (group, head, chunk), groups in order, then heads, then chunks.
__device__ __forceinline__ int att_total(const MegaArgs& m, const int* g_kmax, int n_groups) {
  int total = 0;
  for (int g = 0; g < n_groups; ++g) total += m.H * ((g_kmax[g] + m.aa.CH - 1) / m.aa.CH);
  return total;
}
// This CTA's attention items: a contiguous range of the item order (g, h, c), so that a
// CTA's consecutive items are mostly consecutive chunks of one (group, head).
__device__ __forceinline__ void att_range(int total, int G, int cta, int& i0, int& i1) {
  i0 = (int)((long long)cta * total / G);
  i1 = (int)((long long)(cta + 1) * total / G);
}
__device__ __forceinline__ void att_decode(const MegaArgs& m, const int* g_kmax, int n_groups, int item, int& g, int& h, int& c) {
  int rem = item;
  for (g = 0; g < n_groups; ++g) {
    const int nch = (g_kmax[g] + m.aa.CH - 1) / m.aa.CH;
    if (rem < m.H * nch) {
      h = rem / nch;
      c = rem % nch;
      return;
    }
    rem -= m.H * nch;
  }
  g = 0, h = 0, c = 0;
}
// ---------------------------------------------------------------------------- shared memory
struct MegaSmem {
  unsigned char* ring;
  uint64_t* full;
  uint64_t* empty;
  float* red;    // [kMaxPieces][8][16][RB]; the attention scratch aliases it
  float* ssr;    // [8][RB]
  float* hpre;   // [kMaxPieces][rows][16] epilogue residual inputs
  float* cpre;   // [kMaxPieces][rows][16] cross terms of the next layer (W2)
  float* gain;   // [d] the phase's norm gain; warp w's k-steps written and read by warp w only
  float* qs;     // [rows][DH]
  float* ps;     // [rows][CH]
  float* mrow;
  float* lrow;
  int* lim;
  int* plan_sh;
  int* misc;
  int* rseq;  // this pass's row metadata
  int* rpos;
  int* rlat;
  int* rbyte;
  int* rnkeys;
  int* rpage;    // KV page of each row's position (-1: none)
  float* rope_c; // [rows][dh/2] rotary factors of each row's position
  float* rope_s;
  int* gmeta;  // [5][kMegaRows + 1]: g_seq, g_row0, g_nrows, g_kmax, g_fresh
  int* ppages;  // [16] the producer's KV-page lookups (next item, current item)
  int n_rows, n_groups;
};

// ---------------------------------------------------------------------------- producer
template <int PL, int DH, typename KVT>
__device__ void mega_producer(const MegaArgs& m, MegaSmem& sm, int lane) {
  const int G = gridDim.x, cta = blockIdx.x;
  const uint64_t pol = l2_evict_first();
  unsigned it = 0;
  bool ok = true;
  int gk[kMegaRows + 1], gs[kMegaRows + 1], gf[kMegaRows + 1];  // group kmax, sequence, fresh (lane 0)
  int ng = 0;
  auto load_groups = [&]() {
    ng = min(__ldcg(m.rows.n_groups), kMegaRows);
    for (int g = 0; g < ng; ++g) {
      gk[g] = __ldcg(m.rows.g_kmax + g);
      gs[g] = __ldcg(m.rows.g_seq + g);
      gf[g] = __ldcg(m.rows.g_fresh + g);
    }
  };
  auto next_slot = [&](unsigned bytes) -> unsigned char* {  // lane 0: a free slot armed for `bytes`
    const int slot = it % kRingSlots;
    if (!wait_mbar(m, sm.empty + slot, ((it / kRingSlots) & 1) ^ 1)) {
      ok = false;
      return nullptr;
    }
    mbar_expect_tx(sm.full + slot, bytes);
    ++it;
    return sm.ring + (size_t)slot * kSlotBytes;
  };
  auto issue_phase = [&](const Phase& p) {
    const unsigned tile_bytes = 512u * PL;
    for (int i = 0; i < p.a.count && ok; ++i) {
      const int u = p.a.first + i * p.a.step;
      const unsigned char* src = reinterpret_cast<const unsigned char*>(p.w) +
                                 ((size_t)u * p.ksteps + (size_t)p.seg * p.seg_steps) * tile_bytes;
      const int tps = tiles_per_slot<PL>();
      for (int t0 = 0; t0 < p.seg_steps && ok; t0 += tps) {
        const unsigned bytes = (unsigned)min(tps, p.seg_steps - t0) * tile_bytes;
        unsigned char* dst = next_slot(bytes);
        if (dst) tma_1d(dst, src + (size_t)t0 * tile_bytes, bytes, sm.full + ((it - 1) % kRingSlots), pol);
      }
    }
  };
  auto issue_attention = [&](int layer) {
    const int total = att_total(m, gk, ng);
    const int CH = m.aa.CH, PT = m.ga.PT;
    const unsigned page_bytes = (unsigned)(PT * DH * sizeof(KVT));
    int i0, i1;
    att_range(total, G, cta, i0, i1);
    // the page-table entries of an item are loaded one item ahead: their latency passes
    // while the previous item waits for its slot
    int g = 0, h = 0, c = 0, np = 0;
    int* pages = sm.ppages;  // [2][8] in shared memory: the next item's, then the current item's
    auto lookup = [&](int item) {
      att_decode(m, gk, ng, item, g, h, c);
      const int t0 = c * CH;
      const int tc = min(min(t0 + CH, gk[g]), gf[g]);  // cached keys of this chunk: [t0, tc)
      np = tc > t0 ? (tc - t0 + PT - 1) / PT : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int pi = t0 / PT + j;
        pages[j] = (j < np && pi < m.ga.max_pages) ? __ldcg(m.ga.page_table + gs[g] * m.ga.max_pages + pi) : -1;
      }
    };
    if (i0 < i1) lookup(i0);
    for (int item = i0; item < i1 && ok; ++item) {
      const int ih = h, inp = np;
      int* ipages = pages + 8;
#pragma unroll
      for (int j = 0; j < 8; ++j) ipages[j] = pages[j];
      if (item + 1 < i1) lookup(item + 1);
      int nvalid = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) nvalid += (j < inp && ipages[j] >= 0);
      unsigned char* dst = next_slot(2u * nvalid * page_bytes);
      if (!dst) break;
      uint64_t* bar = sm.full + ((it - 1) % kRingSlots);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j >= inp || ipages[j] < 0) continue;
        const size_t hoff = (((size_t)ipages[j] * m.L + layer) * 2) * m.H;
        const KVT* kv = static_cast<const KVT*>(m.ga.kv);
        const KVT* ksrc = kv + ((hoff + 0 * m.H + ih) * PT) * DH;
        const KVT* vsrc = kv + ((hoff + 1 * m.H + ih) * PT) * DH;
        tma_1d_plain(dst + (size_t)j * page_bytes, ksrc, page_bytes, bar);
        tma_1d_plain(dst + (size_t)CH * DH * sizeof(KVT) + (size_t)j * page_bytes, vsrc, page_bytes, bar);
      }
    }
  };
  if (lane == 0) {
    load_groups();
    for (int pass = 0; pass < m.max_passes && ok; ++pass) {
      for (int l = 0; l < m.L && ok; ++l) {
        issue_phase(phase_of(m, PH_QKV, l, cta, G));
        if (pass > 0 && l == 0) {
          // weights of the next pass went out already; the items need its plan
          if (!wait_flag(m, m.flags + 0, epoch(m, pass - 1, m.L, ST_LOGIT), true)) {
            ok = false;
            break;
          }
          if (__ldcg(m.dec_val) == 0u) break;
          fence_proxy_async_global();
          load_groups();
        }
        issue_attention(l);
        issue_phase(phase_of(m, PH_O, l, cta, G));
        issue_phase(phase_of(m, PH_W13, l, cta, G));
        issue_phase(phase_of(m, PH_W2, l, cta, G));
      }
      if (!ok) break;
      if (pass > 0 && __ldcg(m.dec_val) == 0u) break;
      issue_phase(phase_of(m, PH_HEAD, 0, cta, G));
    }
    // leave no copy in flight: every issued slot must have landed
    const unsigned from = it > (unsigned)kRingSlots ? it - kRingSlots : 0;
    const unsigned long long t0 = gtimer();
    for (unsigned j = from; j < it; ++j)
      while (!mbar_try(sm.full + j % kRingSlots, (j / kRingSlots) & 1) && gtimer() - t0 < 2ull * m.wait_ns + 1000000ull) {
      }
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------- consumer: GEMV phases
// Input row of a phase before the gain, read as exchange words: x[row][col0 + k].
struct XSrc {
  const u64* x;  // NULL: layer-0 input embed[byte] + c_0
  int ld, col0;
  unsigned e;
};

// Wait for and load this warp's k-steps (warp, warp + 8, ...; nkw of them) of
// every live row as B fragments, plus the lanes' sums of squares (canonical
// order).  Rows >= nr get zeros.  A lane loads all its words in one round
// (a dead row reads row 0 and a k-step past nkw re-reads the last one: both
// are always written, never used) and reloads the round only if a word is not
// ready yet -- rare once the sentinels have passed.
template <int NG>
__device__ __forceinline__ bool gather_frags(const MegaArgs& m, const MegaSmem& sm, const XSrc& xs, int nr, int nkw, const float* gain,
                                             uint4 (&xf)[8][NG], float (&ss)[NG], int warp, int lane, int pass) {
  const int g = lane >> 2, t = lane & 3;
  float2 xa[8][NG], xb[8][NG];
  bool ok = true;
  if (!xs.x) {  // layer 0: embedding + cross term, finished data
#pragma unroll
    for (int n = 0; n < NG; ++n) {
      const int row = n * 8 + g;
      const bool live = row < nr;
      const int rr = live ? row : 0;
      const float* e = m.ga.embed + (size_t)sm.rbyte[rr] * m.d;
      const float* c = c_row(m.ga.c_lat, m.ga.max_lat, m.L, 0, m.d, sm.rseq[rr], sm.rlat[rr]);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int k0 = (warp + 8 * min(j, nkw - 1)) * 16 + 2 * t;
        const float2 a = make_float2(__ldg(e + k0) + __ldcg(c + k0), __ldg(e + k0 + 1) + __ldcg(c + k0 + 1));
        const float2 b = make_float2(__ldg(e + k0 + 8) + __ldcg(c + k0 + 8), __ldg(e + k0 + 9) + __ldcg(c + k0 + 9));
        xa[j][n] = (live && j < nkw) ? a : make_float2(0.f, 0.f);
        xb[j][n] = (live && j < nkw) ? b : make_float2(0.f, 0.f);
      }
    }
  } else {
    Spin spins;
    {
      // Sentinels: lane j < nkw polls one word of k-step warp + 8 j (its last column) until
      // every k-step of the warp has data; only then do all lanes load everything.  While waiting,
      // a warp issues at most 8 loads per round.
      // (row blockIdx mod nr: the CTAs' polls spread over the rows instead of meeting on row 0's words)
      const u64* sp = xs.x + (size_t)(blockIdx.x % nr) * xs.ld + xs.col0 + (warp + 8 * min(lane, 7)) * 16 + 15;
      bool ready = lane >= nkw;
      while (true) {
        if (!ready) ready = xw_ok(xw_ld(sp), xs.e);
        if (__all_sync(0xffffffffu, ready)) break;
        if (!spin_step(m, spins)) {
          ok = false;
          break;
        }
      }
    }
    trace_mark(m, pass, TR_SENT << 8);
#pragma unroll
    for (int n = 0; n < NG; ++n) {
      const int row = n * 8 + g;
      const bool live = row < nr;
      const u64* base = xs.x + (size_t)(live ? row : 0) * xs.ld + xs.col0 + 2 * t;
      while (ok) {
        u64 wa[8][2], wb[8][2];
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) xw_ld2(base + (warp + 8 * min(j, nkw - 1)) * 16 + 8 * hf, wa[j][hf], wb[j][hf]);
        bool all = true;
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) all = all && xw_ok(wa[j][hf], xs.e) && xw_ok(wb[j][hf], xs.e);
        if (all) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const bool use = live && j < nkw;
            xa[j][n] = use ? make_float2(xw_val(wa[j][0]), xw_val(wb[j][0])) : make_float2(0.f, 0.f);
            xb[j][n] = use ? make_float2(xw_val(wa[j][1]), xw_val(wb[j][1])) : make_float2(0.f, 0.f);
          }
          break;
        }
        if (!spin_step(m, spins)) ok = false;
      }
      if (!ok) {
#pragma unroll
        for (int j = 0; j < 8; ++j) xa[j][n] = xb[j][n] = make_float2(0.f, 0.f);
      }
    }
  }
  trace_mark(m, pass, TR_GATH << 8);
  const bool norm = gain != nullptr;
  if (norm) {  // the warp's gain values, copied in before the wait (stage_gain)
    cp_async_wait<0>();
    __syncwarp();
  }
#pragma unroll
  for (int n = 0; n < NG; ++n) ss[n] = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float4 gv = make_float4(1.f, 1.f, 1.f, 1.f);
    const int k0 = (warp + 8 * j) * 16 + 2 * t;
    if (norm && j < nkw) gv = make_float4(sm.gain[k0], sm.gain[k0 + 1], sm.gain[k0 + 8], sm.gain[k0 + 9]);
#pragma unroll
    for (int n = 0; n < NG; ++n) {
      const float2 a = xa[j][n], b = xb[j][n];
      if (norm && j < nkw) ss[n] = ss_add(ss[n], a.x, a.y, b.x, b.y);
      const XFrag f = make_xfrag(a.x * gv.x, a.y * gv.y, b.x * gv.z, b.y * gv.w);
      xf[j][n] = make_uint4(f.b0h, f.b1h, f.b0l, f.b1l);
    }
  }
  return ok;
}

// The norm gain of this warp's k-steps (warp + 8 j, j < nkw) into shared memory
// by asynchronous copies, one 16-byte piece per lane, issued before the phase's
// input wait so that their latency hides behind it.
__device__ __forceinline__ void stage_gain(const MegaSmem& sm, const float* gain, int nkw, int warp, int lane) {
  const int j = lane >> 2, o = (warp + 8 * j) * 16 + 4 * (lane & 3);
  if (j < nkw) cp_async16(sm.gain + o, gain + o, 16);
  cp_async_commit();
}

// Epilogue side inputs, into smem before the MMAs: the residual the output is
// added to (O: the stream after the previous layer; W2 finisher: after O) and
// the next layer's cross term (W2 finisher).
template <int NG>
__device__ __forceinline__ bool prefetch_side(const MegaArgs& m, MegaSmem& sm, const Phase& p, int jv0, int nu, int pass, int nr, int tid) {
  const int l = p.layer, d = m.d;
  const bool is_o = p.kind == PH_O;
  const bool fin = p.kind == PH_W2 && p.seg == n_w2_segments(m) - 1;
  if (!is_o && !fin) return true;
  const int n = nu * kMegaRows * 16;
  auto col_of = [&](int i) { return (p.a.first + (jv0 + i / (kMegaRows * 16)) * p.a.step) * 16 + i % 16; };
  auto row_of = [&](int i) { return (i / 16) % kMegaRows; };
  if (fin)
    for (int i = tid; i < n; i += 256) {
      const int row = row_of(i);
      sm.cpre[i] = (l + 1 < m.L && row < nr)
                       ? __ldcg(c_row(m.ga.c_lat, m.ga.max_lat, m.L, l + 1, d, sm.rseq[row], sm.rlat[row]) + col_of(i))
                       : 0.f;
    }
  if (is_o && l == 0) {  // the stream before layer 0 is embed + c_0
    for (int i = tid; i < n; i += 256) {
      const int row = row_of(i);
      sm.hpre[i] = row < nr ? __ldg(m.ga.embed + (size_t)sm.rbyte[row] * d + col_of(i)) +
                                  __ldcg(c_row(m.ga.c_lat, m.ga.max_lat, m.L, 0, d, sm.rseq[row], sm.rlat[row]) + col_of(i))
                            : 0.f;
    }
    return true;
  }
  const unsigned e = is_o ? epoch(m, pass, l - 1, ST_HW) : epoch(m, pass, l, ST_HO);
  // dead rows read row 0's word (always written) and are never used
  return poll_words<kMaxPieces * kMegaRows * 16 / 256>(
      m, n, e, tid, [&](int i) { return m.x_h + (size_t)(row_of(i) < nr ? row_of(i) : 0) * d + col_of(i); },
      [&](int i, float v) { sm.hpre[i] = v; });
}

// Output pair (tile rows r16, r16 + 8) of unit u for row `row`.
template <int NG>
__device__ __forceinline__ bool mega_epilogue(const MegaArgs& m, const MegaSmem& sm, const Phase& p, int jv, int u, int r16, int row,
                                              float v0, float v1, int pass) {
  const int d = m.d, l = p.layer;
  switch (p.kind) {
    case PH_QKV: {
      const unsigned e = epoch(m, pass, l, ST_QKV);
      const GemmArgs& a = m.ga;
      const int tiles_sec = d / 16;
      const int sec = u / tiles_sec, lt = u % tiles_sec;
      const int pos = sm.rpos[row];
      if (sec < 2) {  // q and k tiles hold rotary pairs (j, j + dh/2) in rows (r16, r16 + 8)
        const int tph = m.dh / 16;
        const int h = lt / tph, j = (lt % tph) * 8 + r16;
        const int half = m.dh / 2;
        const float c = sm.rope_c[row * 32 + j], s = sm.rope_s[row * 32 + j];
        const float o0 = v0 * c - v1 * s, o1 = v1 * c + v0 * s;
        const size_t xo = (size_t)row * d + h * m.dh + j;
        if (sec == 0) {
          xw_st(m.x_q + xo, o0, e);
          xw_st(m.x_q + xo + half, o1, e);
          return true;
        }
        const int page = sm.rpage[row];
        float r0 = o0, r1 = o1;
        if (page < 0) {
          set_status(a.status, kErrDevice);
        } else {
          kv_store(a, kv_offset(a, page, l, 0, h, pos % a.PT, kv_dim(a, pos, j)), o0);
          kv_store(a, kv_offset(a, page, l, 0, h, pos % a.PT, kv_dim(a, pos, j + half)), o1);
        }
        if (!a.kv_f32) {
          r0 = __bfloat162float(__float2bfloat16_rn(o0));
          r1 = __bfloat162float(__float2bfloat16_rn(o1));
        }
        xw_st(m.x_k + xo, r0, e);
        xw_st(m.x_k + xo + half, r1, e);
      } else {
        const int n0 = lt * 16 + r16, n1 = n0 + 8;
        const int page = sm.rpage[row];
        if (page < 0) {
          set_status(a.status, kErrDevice);
        } else {
          kv_store(a, kv_offset(a, page, l, 1, n0 / a.dh, pos % a.PT, kv_dim(a, pos, n0 % a.dh)), v0);
          kv_store(a, kv_offset(a, page, l, 1, n1 / a.dh, pos % a.PT, kv_dim(a, pos, n1 % a.dh)), v1);
        }
        float r0 = v0, r1 = v1;
        if (!a.kv_f32) {
          r0 = __bfloat162float(__float2bfloat16_rn(v0));
          r1 = __bfloat162float(__float2bfloat16_rn(v1));
        }
        xw_st(m.x_v + (size_t)row * d + n0, r0, e);
        xw_st(m.x_v + (size_t)row * d + n1, r1, e);
      }
      return true;
    }
    case PH_O: {
      if (m.stall_test && pass == 0 && l == 0 && u == 0) return true;  // test only: never publish
      const unsigned e = epoch(m, pass, l, ST_HO);
      const float* hp = sm.hpre + (jv * kMegaRows + row) * 16;
      xw_st(m.x_h + (size_t)row * d + u * 16 + r16, hp[r16] + v0, e);
      xw_st(m.x_h + (size_t)row * d + u * 16 + r16 + 8, hp[r16 + 8] + v1, e);
      return true;
    }
    case PH_W13: {
      xw_st(m.x_act + (size_t)row * m.F + u * 8 + r16, silu(v0) * v1, epoch(m, pass, l, ST_ACT));
      return true;
    }
    case PH_W2: {
      const int nseg = n_w2_segments(m);
      if (p.seg < nseg - 1) {
        const unsigned e = epoch(m, pass, l, ST_W2P);
        u64* dst = m.x_w2p + ((size_t)p.seg * kMegaRows + row) * d + u * 16 + r16;
        xw_st(dst, v0, e);
        xw_st(dst + 8, v1, e);
        return true;
      }
      // finisher: the segment sums in order, then the residual and the next layer's cross term
      float t0 = v0, t1 = v1;
      bool ok = true;
      if (nseg > 1) {
        constexpr int kMaxSeg = 4;  // d_ffn <= 4096
        const unsigned e = epoch(m, pass, l, ST_W2P);
        float sv[2 * (kMaxSeg - 1)];
        unsigned pending = (1u << (2 * (nseg - 1))) - 1u;
        Spin spins;
        while (pending) {
          u64 w[2 * (kMaxSeg - 1)];
#pragma unroll
          for (int i = 0; i < 2 * (kMaxSeg - 1); ++i)
            if ((pending >> i) & 1u) w[i] = xw_ld(m.x_w2p + ((size_t)(i >> 1) * kMegaRows + row) * d + u * 16 + r16 + 8 * (i & 1));
#pragma unroll
          for (int i = 0; i < 2 * (kMaxSeg - 1); ++i)
            if (((pending >> i) & 1u) && xw_ok(w[i], e)) {
              sv[i] = xw_val(w[i]);
              pending &= ~(1u << i);
            }
          if (pending && !spin_step(m, spins)) {
            ok = false;
            break;
          }
        }
        float a0 = sv[0], a1 = sv[1];
#pragma unroll
        for (int q = 1; q < kMaxSeg - 1; ++q)
          if (q < nseg - 1) {
            a0 = a0 + sv[2 * q];
            a1 = a1 + sv[2 * q + 1];
          }
        t0 = a0 + v0;
        t1 = a1 + v1;
      }
      const float* hp = sm.hpre + (jv * kMegaRows + row) * 16;
      const float* cp = sm.cpre + (jv * kMegaRows + row) * 16;
      float h0 = hp[r16] + t0, h1 = hp[r16 + 8] + t1;
      if (l + 1 < m.L) {
        h0 = h0 + cp[r16];
        h1 = h1 + cp[r16 + 8];
      }
      const unsigned e = epoch(m, pass, l, ST_HW);
      xw_st(m.x_h + (size_t)row * d + u * 16 + r16, h0, e);
      xw_st(m.x_h + (size_t)row * d + u * 16 + r16 + 8, h1, e);
      return ok;
    }
    default: {
      const unsigned e = epoch(m, pass, m.L, ST_LOGIT);
      xw_st(m.x_logit + (size_t)row * 256 + u * 16 + r16, v0, e);
      xw_st(m.x_logit + (size_t)row * 256 + u * 16 + r16 + 8, v1, e);
      return true;
    }
  }
}

// One GEMV phase of this CTA: gather the input once, run its pieces from the
// ring (all eight warps on every piece, warp w on the k-steps = w mod 8 --
// lane group w of the canonical order), reduce across warps in order, apply
// the epilogue.  `it`: ring slots consumed so far.
template <int NG, int PL>
__device__ bool run_gemv(const MegaArgs& m, MegaSmem& sm, const Phase& p, const XSrc& xs, const float* gain, int pass, unsigned& it,
                         int tid) {
  constexpr int RB = 8 * NG;
  if (p.a.count == 0) return true;
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int nr = sm.n_rows;
  const int nkw = (p.seg_steps - warp + 7) / 8;
  trace_mark(m, pass, TR_PH << 8 | p.kind);
  if (gain) stage_gain(sm, gain, nkw, warp, lane);
  // the epilogue's side inputs are older data: fetch them while the phase input is still on its way
  bool ok = prefetch_side<NG>(m, sm, p, 0, min(kMaxPieces, p.a.count), pass, nr, tid);
  trace_mark(m, pass, TR_PRE << 8 | p.kind);
  uint4 xf[8][NG];
  float ss[NG];
  ok = gather_frags<NG>(m, sm, xs, nr, nkw, gain, xf, ss, warp, lane, pass) && ok;
  const bool norm = gain != nullptr;
  if (norm) {
#pragma unroll
    for (int n = 0; n < NG; ++n) {
      float v = ss[n];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      if (t == 0) sm.ssr[warp * RB + n * 8 + g] = v;
    }
  }
  trace_mark(m, pass, TR_IN << 8 | p.kind);
  const int nsl = piece_slots<PL>(p.seg_steps);
  const unsigned tile_bytes = 512u * PL;
  for (int jv0 = 0; jv0 < p.a.count; jv0 += kMaxPieces) {
    const int nu = min(kMaxPieces, p.a.count - jv0);
    if (jv0 > 0) ok = prefetch_side<NG>(m, sm, p, jv0, nu, pass, nr, tid) && ok;
    float acc[kMaxPieces][NG][4];
#pragma unroll
    for (int jv = 0; jv < kMaxPieces; ++jv)
#pragma unroll
      for (int n = 0; n < NG; ++n) acc[jv][n][0] = acc[jv][n][1] = acc[jv][n][2] = acc[jv][n][3] = 0.f;
    if constexpr (PL == 1) {
      // one slot per piece: wait for the group's slots, then walk the k-steps with the pieces
      // interleaved, so that their MMA chains overlap (each chain is the same as run alone)
      constexpr int TPW = kSlotBytes / 512 / 8;  // tiles of a slot per warp
      uint32_t stage[kMaxPieces];  // this lane's address in each piece's slot (shared memory)
#pragma unroll
      for (int jv = 0; jv < kMaxPieces; ++jv) {
        stage[jv] = smem_u32(sm.ring) + lane * 16 + warp * 512;
        if (jv < nu) {
          const unsigned itu = it + jv;
          const int slot = itu % kRingSlots;
          if (!wait_mbar(m, sm.full + slot, (itu / kRingSlots) & 1)) ok = false;
          stage[jv] += slot * kSlotBytes;
        }
      }
      trace_mark(m, pass, TR_MW << 8);
      const int ntiles = p.seg_steps;  // <= 64: one slot
      auto chains = [&](auto nu_c) {
        constexpr int NU = decltype(nu_c)::value;
#pragma unroll
        for (int q = 0; q < TPW; ++q) {
          if (8 * q + warp < ntiles) {  // k-step 8 q + warp of every piece
            uint4 w[NU][1];
#pragma unroll
            for (int jv = 0; jv < NU; ++jv) w[jv][0] = lds128(stage[jv] + q * 4096);
#pragma unroll
            for (int n = 0; n < NG; ++n) {
              const XFrag xq{xf[q][n].x, xf[q][n].y, xf[q][n].z, xf[q][n].w};
#pragma unroll
              for (int jv = 0; jv < NU; ++jv) mma_step<1>(acc[jv][n], w[jv], xq);
            }
          }
        }
      };
      if (nu == 1) chains(std::integral_constant<int, 1>{});
      else if (nu == 2) chains(std::integral_constant<int, 2>{});
      else if (nu == 3) chains(std::integral_constant<int, 3>{});
      else chains(std::integral_constant<int, 4>{});
      __syncwarp();
      if (lane == 0)
#pragma unroll
        for (int jv = 0; jv < kMaxPieces; ++jv)
          if (jv < nu) mbar_arrive(sm.empty + (it + jv) % kRingSlots);
      it += nu;
    } else {
#pragma unroll
      for (int jv = 0; jv < kMaxPieces; ++jv) {
        if (jv < nu) {
          constexpr int TPS = kSlotBytes / (512 * PL);           // tiles per slot
          constexpr int TPW = TPS / 8;                           // tiles of a slot per warp
          constexpr int MAXSL = (kSegSteps + TPS - 1) / TPS;     // slots per piece at most
#pragma unroll
          for (int sl = 0; sl < MAXSL; ++sl) {
            if (sl < nsl) {
              const unsigned itu = it++;
              const int slot = itu % kRingSlots;
              if (!wait_mbar(m, sm.full + slot, (itu / kRingSlots) & 1)) ok = false;
              trace_mark(m, pass, TR_MW << 8 | (jv * MAXSL + sl));
              const unsigned char* stage = sm.ring + (size_t)slot * kSlotBytes;
              const int ntiles = min(TPS, p.seg_steps - sl * TPS);
              uint4 w[TPW][PL];
#pragma unroll
              for (int q = 0; q < TPW; ++q)
#pragma unroll
                for (int pl = 0; pl < PL; ++pl)
                  w[q][pl] = *reinterpret_cast<const uint4*>(stage + (size_t)min(8 * q + warp, ntiles - 1) * tile_bytes + pl * 512 + lane * 16);
#pragma unroll
              for (int q = 0; q < TPW; ++q) {
                const int j = sl * TPW + q;  // this warp's j-th k-step of the piece: k-step 8 j + warp
                if (8 * q + warp < ntiles)
#pragma unroll
                  for (int n = 0; n < NG; ++n)
                    mma_step<PL>(acc[jv][n], w[q], XFrag{xf[j][n].x, xf[j][n].y, xf[j][n].z, xf[j][n].w});
              }
              __syncwarp();
              if (lane == 0) mbar_arrive(sm.empty + slot);
            }
          }
        }
      }
    }
    trace_mark(m, pass, TR_MMA << 8 | p.kind);
#pragma unroll
    for (int jv = 0; jv < kMaxPieces; ++jv) {
      if (jv < nu) {
        float* rw = sm.red + (size_t)(jv * 8 + warp) * 16 * RB;
#pragma unroll
        for (int n = 0; n < NG; ++n) {
          const int c = n * 8 + 2 * t;
          rw[g * RB + c] = acc[jv][n][0];
          rw[g * RB + c + 1] = acc[jv][n][1];
          rw[(g + 8) * RB + c] = acc[jv][n][2];
          rw[(g + 8) * RB + c + 1] = acc[jv][n][3];
        }
      }
    }
    consumer_sync();
    for (int pi = tid; pi < nu * 8 * RB; pi += 256) {
      const int jv = pi / (8 * RB), q = pi % (8 * RB);
      const int r16 = q & 7, col = q >> 3;
      if (col >= nr) continue;
      const float* ru = sm.red + (size_t)jv * 8 * 16 * RB;
      float v0 = ru[r16 * RB + col], v1 = ru[(r16 + 8) * RB + col];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) {
        v0 += ru[(w * 16 + r16) * RB + col];
        v1 += ru[(w * 16 + r16 + 8) * RB + col];
      }
      float rs = 1.0f;
      if (norm) {
        float sv = sm.ssr[col];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) sv += sm.ssr[w * RB + col];
        rs = 1.0f / sqrtf(sv / (float)(p.ksteps * 16) + m.eps);
      }
      const int u = p.a.first + (jv0 + jv) * p.a.step;
      ok = mega_epilogue<NG>(m, sm, p, jv, u, r16, col, v0 * rs, v1 * rs, pass) && ok;
    }
    consumer_sync();  // red, hpre, cpre free again
  }
  trace_mark(m, pass, TR_DONE << 8 | p.kind);
  return ok;
}

// ---------------------------------------------------------------------------- consumer: attention
// attn_combine for one (row, head) by one warp, with the chunk partials read as
// exchange words.  Each chunk's (m, l) pair and each pair of o columns is one
// 16-byte load (a record is 2 + DH words, so both start on 16 bytes).  Lane j
// holds chunk j of each 32-chunk block for the weights; lane c owns columns
// 2c and 2c + 1 and reads eight chunks per round of loads.  The arithmetic is
// attn_combine's, in the same order: the maximum over chunks with l > 0, the
// lanes' l sums then a warp sum, and per column one fmaf chain in chunk order.
template <int DH>
__device__ __forceinline__ bool combine_row_xw(const MegaArgs& m, const u64* base, int nch, int lane, unsigned e, u64* out, unsigned e_out,
                                               int pass) {
  static_assert(DH == 32 || DH == 64, "column pairs per lane");
  constexpr int REC = 2 + DH;
  constexpr int RND = 5;  // chunks per round of loads (more spills registers)
  const bool col_ok = 2 * lane < DH;
  bool ok = true;
  auto poll_ml = [&](int ch, float& mm, float& ll) {
    Spin spins;
    while (true) {
      u64 a, b;
      xw_ld2(base + (size_t)ch * REC, a, b);
      if (xw_ok(a, e) && xw_ok(b, e)) {
        mm = xw_val(a), ll = xw_val(b);
        return true;
      }
      if (!spin_step(m, spins)) return false;
    }
  };
  float mmax = -INFINITY;
  float m0 = 0.f, l0 = 0.f;  // the lane's chunk of the first block, kept for the second pass
#pragma unroll 1
  for (int ch = lane; ch < nch; ch += 32) {
    float mm = 0.f, ll = 0.f;
    ok = poll_ml(ch, mm, ll) && ok;
    if (ch < 32) m0 = mm, l0 = ll;
    if (ll > 0.f) mmax = fmaxf(mmax, mm);
  }
  mmax = warp_max(mmax);
  trace_mark(m, pass, TR_CML << 8);
  float l = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll 1
  for (int cb = 0; cb < nch; cb += 32) {
    const int nb = min(32, nch - cb);
    float w = 0.f;
    if (cb + lane < nch) {
      float mm = m0, ll = l0;
      if (cb > 0) ok = poll_ml(cb + lane, mm, ll) && ok;
      if (ll > 0.f) {
        w = expf(mm - mmax);
        l = fmaf(ll, w, l);
      }
    }
#pragma unroll 1
    for (int sb = 0; sb < nb; sb += RND) {
      const u64* p = base + (size_t)(cb + sb) * REC + 2 + 2 * lane;
      unsigned pending = 0;
#pragma unroll
      for (int j = 0; j < RND; ++j)
        if (sb + j < nb && col_ok) pending |= 1u << j;
      u64 va[RND], vb[RND];
      Spin spins;
      while (true) {
#pragma unroll
        for (int j = 0; j < RND; ++j)  // every load of the round first, then the checks
          if ((pending >> j) & 1u) xw_ld2(p + (size_t)j * REC, va[j], vb[j]);
        unsigned bad = 0;
#pragma unroll
        for (int j = 0; j < RND; ++j)
          if (((pending >> j) & 1u) && (!xw_ok(va[j], e) || !xw_ok(vb[j], e))) bad |= 1u << j;
        pending = bad;
        if (!pending) break;
        if (!spin_step(m, spins)) {
          ok = false;
          break;
        }
      }
      trace_mark(m, pass, TR_CSUB << 8);
#pragma unroll
      for (int j = 0; j < RND; ++j) {
        const float wj = __shfl_sync(0xffffffffu, w, (sb + j) & 31);
        if (sb + j < nb) {
          o0 = fmaf(xw_val(va[j]), wj, o0);
          o1 = fmaf(xw_val(vb[j]), wj, o1);
        }
      }
    }
  }
  l = warp_sum(l);
  if (col_ok) {
    xw_st(out + 2 * lane, o0 / l, e_out);
    xw_st(out + 2 * lane + 1, o1 / l, e_out);
  }
  return ok;
}

// This CTA's attention items of layer l, then the combines it owns.
template <int DH, typename KVT>
__device__ bool run_attention(const MegaArgs& m, MegaSmem& sm, int l, int pass, unsigned& it, int tid) {
  const int G = gridDim.x, cta = blockIdx.x;
  const int CH = m.aa.CH, H = m.H, d = m.d;
  const int* gk = sm.gmeta + 3 * (kMegaRows + 1);
  const int ng = sm.n_groups;
  const int total = att_total(m, gk, ng);
  const int warp = tid >> 5, lane = tid & 31;
  // the slot holds whole pages as stored: 64-element bf16 rows keep their permuted pieces
  constexpr int KST = kv_swizzled<DH, KVT>() ? 0 : DH;
  bool ok = true;
  const unsigned e_qkv = epoch(m, pass, l, ST_QKV), e_part = epoch(m, pass, l, ST_PART);
  trace_mark(m, pass, TR_ATT << 8);
  int i0, i1;
  att_range(total, G, cta, i0, i1);
  int qg = -1, qh = -1;  // (group, head) whose queries sm.qs holds
  for (int item = i0; item < i1; ++item) {
    int g, h, c;
    att_decode(m, gk, ng, item, g, h, c);
    const bool new_q = g != qg || h != qh;
    qg = g, qh = h;
    const int row0 = sm.gmeta[1 * (kMegaRows + 1) + g], nr = sm.gmeta[2 * (kMegaRows + 1) + g];
    const int kmax = gk[g], fresh = sm.gmeta[4 * (kMegaRows + 1) + g];
    const int t0 = c * CH, nk = min(CH, kmax - t0);
    const unsigned itu = it++;
    const int slot = itu % kRingSlots;
    KVT* ks = reinterpret_cast<KVT*>(sm.ring + (size_t)slot * kSlotBytes);
    KVT* vs = ks + CH * DH;
    // this pass's keys and values, and q, as exchange words; the cached pages are in the slot
    if (!wait_mbar(m, sm.full + slot, (itu / kRingSlots) & 1)) ok = false;
    trace_mark(m, pass, TR_ISLOT << 8);
    const int f0 = max(t0, fresh), f1 = t0 + nk;
    constexpr int HP = DH / 2;  // column pairs of a head
    const int nfp = f1 > f0 ? (f1 - f0) * HP : 0;  // this pass's keys in the chunk, times HP
    // one poll for this pass's keys and values in the chunk and (for a new (group, head)) the
    // rows' queries, by column pairs
    ok = poll_pairs<(3 * kMegaRows * HP + 255) / 256>(
             m, 2 * nfp + (new_q ? nr * HP : 0), e_qkv, tid,
             [&](int i) {
               const u64* src = m.x_q;
               int r, c;
               if (i < 2 * nfp) {
                 const int sel = i >= nfp, rem = i - sel * nfp;
                 src = sel ? m.x_v : m.x_k;
                 r = row0 + f0 - fresh + rem / HP, c = rem % HP;
               } else {
                 const int q = i - 2 * nfp;
                 r = row0 + q / HP, c = q % HP;
               }
               return src + (size_t)r * d + h * DH + 2 * c;
             },
             [&](int i, float v0, float v1) {
               if (i < 2 * nfp) {
                 const int sel = i >= nfp, rem = i - sel * nfp;
                 KVT* dst = (sel ? vs : ks) + kv_at<KST>(f0 - t0 + rem / HP, 2 * (rem % HP));
                 if constexpr (sizeof(KVT) == 2) {
                   *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(v0, v1);
                 } else {
                   dst[0] = v0;
                   dst[1] = v1;
                 }
               } else {
                 const int q = i - 2 * nfp;
                 *reinterpret_cast<float2*>(sm.qs + 2 * q) = make_float2(v0 * m.aa.scale, v1 * m.aa.scale);
               }
             }) &&
         ok;
    trace_mark(m, pass, TR_IPOLL << 8);
    if (tid < kMegaRows) sm.lim[tid] = (tid < nr) ? sm.rnkeys[row0 + tid] - t0 : 0;
    if constexpr (sizeof(KVT) == 2) {  // zero V rows nk .. next multiple of 16 (read by the last key tile)
      const int pad = ((nk + 15) & ~15) - nk;
      for (int i = tid; i < pad * (DH / 8); i += 256)
        *reinterpret_cast<uint4*>(vs + (size_t)(nk + i / (DH / 8)) * DH + (i % (DH / 8)) * 8) = make_uint4(0, 0, 0, 0);
    }
    consumer_sync();
    u64* part = m.x_part + (((size_t)row0 * H + h) * m.CMAX + c) * (2 + DH);
    const size_t rstride = (size_t)H * m.CMAX * (2 + DH);
    attn_chunk_core<DH, KVT, KST>(
        CH, sm.qs, sm.ps, ks, vs, sm.mrow, sm.lrow, sm.lim, nr, nk, tid, 256, consumer_sync,
        [&](int r, int col, float v) { xw_st(part + r * rstride + 2 + col, v, e_part); },
        [&](int r, float mm, float ll) {
          xw_st(part + r * rstride, mm, e_part);
          xw_st(part + r * rstride + 1, ll, e_part);
        },
        [&](int stage) { trace_mark(m, pass, TR_ISTAGE << 8 | stage); });
    trace_mark(m, pass, TR_ICORE << 8);
    fence_proxy_async_smem();  // the slot was written by these threads; the producer refills it by bulk copy
    consumer_sync();
    if (lane == 0) mbar_arrive(sm.empty + slot);
  }
  trace_mark(m, pass, TR_ATT_DONE << 8);
  // combines: pair p = g H + h belongs to CTA p mod G; one warp per row
  const unsigned e_att = epoch(m, pass, l, ST_ATT);
  trace_mark(m, pass, TR_CBEG << 8);
  for (int pr = cta; pr < ng * H; pr += G) {
    const int g = pr / H, h = pr % H;
    const int row0 = sm.gmeta[1 * (kMegaRows + 1) + g], nr = sm.gmeta[2 * (kMegaRows + 1) + g];
    for (int r = warp; r < nr; r += kMegaConsumers) {
      const int row = row0 + r;
      const int rnch = (sm.rnkeys[row] + CH - 1) / CH;
      const u64* base = m.x_part + (((size_t)row * H + h) * m.CMAX) * (2 + DH);
      trace_mark(m, pass, TR_CROW << 8);
      ok = combine_row_xw<DH>(m, base, rnch, lane, e_part, m.x_att + (size_t)row * d + h * DH, e_att, pass) && ok;
    }
  }
  trace_mark(m, pass, TR_COMB << 8);
  return ok;
}

// ---------------------------------------------------------------------------- bookkeeping (CTA 0)
// After the head of pass `pass`: statistics, the mode's bookkeeping, the
// decision to go on, the plan of the next pass.
__device__ bool mega_bookkeeping(const MegaArgs& m, MegaSmem& sm, int pass, int nr, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  bool ok = true;
  // every CTA's stores of this pass (the KV cache included) happen before the decision
  if (tid == 0) ok = wait_flag(m, m.flags + 1, (unsigned)(gridDim.x * (pass + 1)), false);
  const unsigned e = epoch(m, pass, m.L, ST_LOGIT);
  for (int half = 0; half < 2; ++half)  // two rounds of at most eight words per thread
    ok = poll_words<kMegaRows / 2>(m, max(0, min(nr, (half + 1) * kMegaRows / 2) - half * kMegaRows / 2) * 256, e, tid,
                                   [&](int i) { return m.x_logit + half * (kMegaRows / 2) * 256 + i; },
                                   [&](int i, float v) { m.logits[half * (kMegaRows / 2) * 256 + i] = v; }) &&
         ok;
  if (tid == 0) sm.misc[1] = 0;
  __threadfence_block();
  ok = consumer_and(ok);
  for (int r = warp; r < nr; r += 8) {
    float c, g, en;
    int p;
    head_stats_row(m.logits + (size_t)r * 256, lane, c, p, g, en);
    if (lane == 0) {
      m.conf[r] = c;
      m.pred[r] = p;
      m.gap[r] = g;
      m.ent[r] = en;
    }
  }
  __threadfence_block();
  consumer_sync();
  int cont = 0;
  if (m.mode == MM_DIFFUSE) {
    for (int s = warp; s < m.batch; s += 8) {
      if (m.sd.active[s]) {
        const bool left =
            unmask_seq(m.sd, s, m.batch, m.k, m.alpha, pass, m.conf, m.pred, m.logits, m.out_logits, lane, m.eb ? m.ent : nullptr);
        if (left && lane == 0) atomicOr(sm.misc + 1, 1);
      }
    }
    consumer_sync();
    cont = sm.misc[1] && pass + 1 < m.max_passes;
  } else if (m.mode == MM_DRAFT_AR) {
    for (int s = warp; s < m.batch; s += 8) draft_ar_seq(m.sd, s, m.batch, pass, m.pred, m.logits, m.out_logits, lane);
    cont = pass + 1 < m.max_passes;
  } else {
    for (int s = warp; s < m.batch; s += 8)
      accept_seq(m.sd, s, m.k, m.pred, m.vlat, m.logits, m.out_acc, m.out_next, m.out_logits, lane);
  }
  __threadfence_block();
  consumer_sync();
  if (cont && ok) {
    PlanArgs p = m.plan;
    if (m.mode == MM_DIFFUSE) {
      p.mode = PL_BLOCK;
    } else {
      p.mode = PL_ARDRAFT;
      p.step = pass + 1;
    }
    plan_rows(p, m.batch, nullptr, nullptr, m.sd, m.rows, tid, 256, sm.plan_sh, consumer_sync);
  }
  consumer_sync();
  if (tid == 0) {
    *(volatile unsigned*)m.dec_val = (cont && ok) ? 1u : 0u;
    __threadfence();
    st_release(m.flags + 0, e);
  }
  return ok;
}

// ---------------------------------------------------------------------------- the kernel
template <int NG, int PL, int DH, typename KVT>
__global__ void __launch_bounds__(kMegaThreads, 1) k_mega(const __grid_constant__ MegaArgs m) {
  extern __shared__ __align__(1024) unsigned char mega_smem[];
  __shared__ uint64_t bars[2 * kRingSlots];
  __shared__ int plan_sh[3 * (kMaxCallBatch + 1)];
  __shared__ int misc[4];
  __shared__ float mrow[kMegaRows], lrow[kMegaRows];
  __shared__ int lim[kMegaRows];
  __shared__ int rmeta[6][kMegaRows];
  __shared__ int gmeta[5 * (kMegaRows + 1)];
  __shared__ float rope_tab[2][kMegaRows * 32];  // dh <= 64
  __shared__ int ppages[16];

  MegaSmem sm;
  sm.ring = mega_smem;
  unsigned char* p = mega_smem + (size_t)kRingSlots * kSlotBytes;
  sm.red = reinterpret_cast<float*>(p);
  sm.qs = sm.red;  // attention scratch aliases the reduction buffer
  sm.ps = sm.qs + kMegaRows * DH;
  p += (size_t)kMaxPieces * 8 * 16 * 8 * NG * 4 > (size_t)(kMegaRows * DH + kMegaRows * 128) * 4
           ? (size_t)kMaxPieces * 8 * 16 * 8 * NG * 4
           : (size_t)(kMegaRows * DH + kMegaRows * 128) * 4;
  sm.ssr = reinterpret_cast<float*>(p);
  p += 8 * 8 * kMegaMaxNG * 4;
  sm.hpre = reinterpret_cast<float*>(p);
  p += kMaxPieces * kMegaRows * 16 * 4;
  sm.cpre = reinterpret_cast<float*>(p);
  p += kMaxPieces * kMegaRows * 16 * 4;
  sm.gain = reinterpret_cast<float*>(p);
  sm.full = bars;
  sm.empty = bars + kRingSlots;
  sm.mrow = mrow;
  sm.lrow = lrow;
  sm.lim = lim;
  sm.plan_sh = plan_sh;
  sm.misc = misc;
  sm.rseq = rmeta[0];
  sm.rpos = rmeta[1];
  sm.rlat = rmeta[2];
  sm.rbyte = rmeta[3];
  sm.rnkeys = rmeta[4];
  sm.rpage = rmeta[5];
  sm.rope_c = rope_tab[0];
  sm.rope_s = rope_tab[1];
  sm.gmeta = gmeta;
  sm.ppages = ppages;

  const int tid = threadIdx.x;
  if (tid == 0) {
    s_trace_n = 0;
    for (int i = 0; i < kRingSlots; ++i) {
      mbar_init(sm.full + i, 1);
      mbar_init(sm.empty + i, kMegaConsumers);
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();

  if (tid >= 256) {  // the producer's warpgroup
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kProducerRegs));
    if (tid < 288) mega_producer<PL, DH, KVT>(m, sm, tid & 31);
    return;
  }
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kConsumerRegs));
  const int G = gridDim.x;
  unsigned it = 0;
  bool ok = true;
  for (int pass = 0; pass < m.max_passes && ok; ++pass) {
    if (pass > 0) {
      if (tid == 0) misc[2] = wait_flag(m, m.flags + 0, epoch(m, pass - 1, m.L, ST_LOGIT), true) ? (int)__ldcg(m.dec_val) : -1;
      consumer_sync();
      const int go = misc[2];
      consumer_sync();
      if (go <= 0) {
        ok = go == 0;
        break;
      }
    }
    // this pass's rows (live rows only; the rest never reach an output)
    sm.n_rows = min(__ldcg(m.rows.n_rows), kMegaRows);
    sm.n_groups = min(__ldcg(m.rows.n_groups), kMegaRows);
    if (tid < kMegaRows) {
      const bool live = tid < sm.n_rows;
      sm.rseq[tid] = live ? __ldcg(m.rows.seq + tid) : 0;
      sm.rpos[tid] = live ? __ldcg(m.rows.pos + tid) : 0;
      sm.rlat[tid] = live ? __ldcg(m.rows.lat + tid) : 0;
      sm.rbyte[tid] = live ? __ldcg(m.rows.byte + tid) : 0;
      sm.rnkeys[tid] = live ? __ldcg(m.rows.nkeys + tid) : 0;
    }
    consumer_sync();
    if (tid < kMegaRows) {  // the KV page of each row's position (dead rows: position 0)
      const int pi = sm.rpos[tid] / m.ga.PT;
      sm.rpage[tid] = (pi < m.ga.max_pages) ? __ldcg(m.ga.page_table + sm.rseq[tid] * m.ga.max_pages + pi) : -1;
    }
    for (int i = tid; i < kMegaRows * (m.dh / 2); i += 256) {  // rotary factors of each row's position
      const int r = i / (m.dh / 2), j = i % (m.dh / 2);
      const size_t src = (size_t)sm.rpos[r] * (m.dh / 2) + j;
      sm.rope_c[r * 32 + j] = __ldg(m.ga.rope_cos + src);
      sm.rope_s[r * 32 + j] = __ldg(m.ga.rope_sin + src);
    }
    if (tid < sm.n_groups) {
      gmeta[0 * (kMegaRows + 1) + tid] = __ldcg(m.rows.g_seq + tid);
      gmeta[1 * (kMegaRows + 1) + tid] = __ldcg(m.rows.g_row0 + tid);
      gmeta[2 * (kMegaRows + 1) + tid] = __ldcg(m.rows.g_nrows + tid);
      gmeta[3 * (kMegaRows + 1) + tid] = __ldcg(m.rows.g_kmax + tid);
      gmeta[4 * (kMegaRows + 1) + tid] = __ldcg(m.rows.g_fresh + tid);
    }
    consumer_sync();
    trace_mark(m, pass, TR_PASS << 8);
    const int nr = sm.n_rows;
    // The pass as one loop of GEMV steps (per layer QKV, O, W13, W2; then the head), so that
    // run_gemv and run_attention are each inlined once: the kernel's code stays small enough
    // for the instruction caches to keep a phase's working set.
    const int nsteps = 4 * m.L + 1;
    for (int st = 0; st < nsteps && ok; ++st) {
      const int l = st >> 2, k = st & 3;
      XSrc xs;
      xs.ld = m.d, xs.col0 = 0;
      const float* gain = nullptr;
      Phase ph;
      if (l == m.L) {  // the byte head
        ph = phase_of(m, PH_HEAD, 0, blockIdx.x, G);
        xs.x = m.x_h, xs.e = epoch(m, pass, m.L - 1, ST_HW), gain = m.final_norm;
      } else if (k == 0) {
        ph = phase_of(m, PH_QKV, l, blockIdx.x, G);
        xs.x = (l == 0) ? nullptr : m.x_h, xs.e = (l == 0) ? 0u : epoch(m, pass, l - 1, ST_HW), gain = m.layers[l].attn_norm;
      } else if (k == 1) {
        ph = phase_of(m, PH_O, l, blockIdx.x, G);
        xs.x = m.x_att, xs.e = epoch(m, pass, l, ST_ATT);
      } else if (k == 2) {
        ph = phase_of(m, PH_W13, l, blockIdx.x, G);
        xs.x = m.x_h, xs.e = epoch(m, pass, l, ST_HO), gain = m.layers[l].ffn_norm;
      } else {
        ph = phase_of(m, PH_W2, l, blockIdx.x, G);
        xs.x = m.x_act, xs.ld = m.F, xs.col0 = ph.seg * kSegCols, xs.e = epoch(m, pass, l, ST_ACT);
      }
      ok = consumer_and(run_gemv<NG, PL>(m, sm, ph, xs, gain, pass, it, tid) && ok);
      if (k == 0 && l < m.L) ok = consumer_and(run_attention<DH, KVT>(m, sm, l, pass, it, tid) && ok);
    }
    if (!ok) break;
    // this CTA's stores of the pass (KV cache included) are done: arrive
    if (tid == 0) {
      __threadfence();
      red_release_add(m.flags + 1, 1u);
    }
    if (!ok) break;
    if (blockIdx.x == 0) ok = consumer_and(mega_bookkeeping(m, sm, pass, nr, tid) && ok);
    trace_mark(m, pass, TR_BOOK << 8);
  }
}

}  // namespace bltdec
