// Persistent decoder-pass kernel: every pass of one C-ABI call (the confidence
// unmasking loop of BLT-D, the k passes of a BLT-S draft, the BLT-DV draft
// loop, or the verification pass) in one cooperative launch, one CTA per SM.
//
// Warp roles: warps 0..7 consume (tensor-core GEMV, attention, bookkeeping),
// warp 8 produces: it streams this CTA's weight tiles for the whole pass
// through a shared-memory ring with 1-D bulk TMA copies, so HBM keeps
// streaming while consumers wait on data dependencies.
//
// Work: each projection is cut into units of 16 output rows (a tile row of
// the fragment-ordered weights).  The units of all phases of a pass
// (QKV, O, W13, W2 per layer, then the byte head) are dealt round-robin to
// the CTAs, continuing across phases, so every CTA streams about the same
// number of bytes at every point of the pass.
//
// Dependencies are per-unit epoch flags in global memory (release store by
// the producing CTA, acquire poll by the consumer), not grid barriers: a
// QKV k-step waits only for the W2 unit that wrote its 16 input columns,
// an O-projection k-step for the attention head it reads, and so on.  Every
// wait is bounded; a wait that runs out sets the abort word and the status,
// and all CTAs leave.  The arithmetic of every unit, attention chunk,
// combine and bookkeeping step is the device code the per-phase kernels use,
// so both paths give bit-identical results.
#pragma once

#include "kernels.cuh"

namespace bltdec {

constexpr int kMegaConsumers = 8;
constexpr int kMegaThreads = (kMegaConsumers + 1) * 32;
constexpr int kStageTiles = 64;                 // k16 tiles of one unit per ring slot
constexpr int kTPW = kStageTiles / 8;           // tiles of a stage per consumer warp
constexpr int kRingBytes = 128 * 1024;          // weight ring
constexpr int kMegaMaxNG = 2;                   // <= 16 rows per pass
constexpr unsigned kSpinLimit = 1u << 26;       // polls before a wait gives up

enum MegaMode : int { MM_DIFFUSE = 0, MM_DRAFT_AR = 1, MM_VERIFY = 2 };

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
  GemmArgs ga;  // epilogue context: pointers shared by all phases
  AttnArgs aa;
  RowsDev rows;
  SeqDev sd;
  float* h;
  float* q;
  float* att;
  float* act;
  float* logits;
  float* conf;
  float* ent;  // per-row entropy of the byte head (EB sampling)
  int eb;      // block unmasking by EB sampling (bound alpha) instead of confidence
  int* pred;
  float* gap;
  unsigned* flags;  // epoch flags, see flag offsets below
  int f_qkv, f_o, f_w13, f_w2, f_head, f_att, f_dec;
  unsigned* attn_cnt;  // [max_groups][H] arrival counters
  unsigned* dec_val;   // continue word written with the decision flag
  unsigned epoch0;
  int* abort;
  unsigned long long* trace;  // debug timestamps [cta][kTraceEvents] of pass 0 (NULL: off)
  int mode, batch, k, max_passes;
  float alpha;
  const int* vlat;
  float* out_logits;
  int* out_acc;
  unsigned char* out_next;
  PlanArgs plan;  // template for the device-side plans of passes >= 2
};

// ---------------------------------------------------------------------------- sync primitives
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint64_t* b, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(b)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_n(uint64_t* b, unsigned n) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(b)), "r"(n) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void tma_1d(void* dst, const void* src, unsigned bytes, uint64_t* b, uint64_t pol) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;\n" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(b)), "l"(pol)
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
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }

// Bounded waits.  Return false when the wait gave up (abort raised).
__device__ __forceinline__ bool wait_flag(const MegaArgs& m, const unsigned* f, unsigned target) {
  unsigned n = 0;
  while ((int)(ld_acquire(f) - target) < 0) {
    if (++n > 64) __nanosleep(64);
    if ((n & 1023) == 0 && *(volatile int*)m.abort) return false;
    if (n > kSpinLimit) {
      atomicExch(m.abort, 1);
      set_status(m.sd.status, kErrDevice);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ bool wait_mbar(const MegaArgs& m, uint64_t* b, unsigned parity) {
  unsigned n = 0;
  while (!mbar_try(b, parity)) {
    if ((++n & 1023) == 0 && *(volatile int*)m.abort) return false;
    if (n > kSpinLimit) {
      atomicExch(m.abort, 1);
      set_status(m.sd.status, kErrDevice);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ unsigned ld_relaxed(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_acquire() { asm volatile("fence.acq_rel.gpu;\n" ::: "memory"); }
__device__ __forceinline__ void fence_acq_rel() { asm volatile("fence.acq_rel.gpu;\n" ::: "memory"); }
__device__ __forceinline__ void st_relaxed(unsigned* p, unsigned v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}

// Warp-wide wait until flag(i) >= target for every i < n: each lane polls
// its share with relaxed loads (all in flight at once), then one acquire
// fence orders the data reads that follow.  Bounded like wait_flag.
template <class FlagFn>
__device__ __forceinline__ bool warp_wait(const MegaArgs& m, int n, FlagFn flag, unsigned target) {
  const int lane = threadIdx.x & 31;
  unsigned spins = 0;
  while (true) {
    bool mine = true;
#pragma unroll 1
    for (int i = lane; i < n; i += 32) mine &= (int)(ld_relaxed(flag(i)) - target) >= 0;
    if (__all_sync(0xffffffffu, mine)) break;
    ++spins;
    if (spins > 8) __nanosleep(128);
    if ((spins & 255) == 0 && *(volatile int*)m.abort) return false;
    if (spins > (kSpinLimit >> 6)) {
      if (lane == 0) {
        atomicExch(m.abort, 1);
        set_status(m.sd.status, kErrDevice);
      }
      return false;
    }
  }
  fence_acquire();
  __syncwarp();
  return true;
}

// Device-side timestamps (debug): trace[cta][event] = %globaltimer.
constexpr int kTraceEvents = 1024;
__shared__ int s_trace_n;  // this CTA's event count of the traced pass (debug only)
// Event word: code << 48 | low 48 bits of %globaltimer.  Recorded by thread 0 in pass 0.
// Compiled in only with -DBLTDEC_MEGA_TRACE (the marks cost instruction-cache space).
__device__ __forceinline__ void trace_mark(const MegaArgs& m, int pass, int code) {
#ifdef BLTDEC_MEGA_TRACE
  if (m.trace && pass == 0 && threadIdx.x == 0) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    const int i = s_trace_n++;
    if (i < kTraceEvents) m.trace[(size_t)blockIdx.x * kTraceEvents + i] = ((unsigned long long)code << 48) | (t & 0xFFFFFFFFFFFFull);
  }
#endif
}
enum TraceCode : int {
  TR_PASS = 1, TR_PHASE_BEGIN = 2, TR_INPUTS = 3, TR_XBUILT = 4, TR_KLOOP = 5, TR_REDUCED = 6, TR_UNIT_DONE = 7,
  TR_ATT_BEGIN = 8, TR_ATT_QKV = 9, TR_ATT_LOADED = 10, TR_ATT_COMPUTED = 11, TR_ATT_DONE = 12, TR_HEAD = 13, TR_BOOK = 14,
  TR_XLOADED = 15, TR_ATT_STEP = 16
};

// ---------------------------------------------------------------------------- schedule
enum PhaseKind : int { PH_QKV = 0, PH_O = 1, PH_W13 = 2, PH_W2 = 3, PH_HEAD = 4 };

struct Phase {
  int kind, layer, units, ksteps, base;
  const uint4* w;
};

// Phase ph of a pass: ph = 4*l + {0: QKV, 1: O, 2: W13, 3: W2}; ph = 4L: head.
__device__ __forceinline__ Phase phase_of(const MegaArgs& m, int ph) {
  Phase p;
  const int L = m.L, d = m.d, F = m.F;
  const int per_layer = 3 * d / 16 + d / 16 + 2 * F / 16 + d / 16;
  p.layer = ph / 4;
  p.base = p.layer * per_layer;
  if (ph >= 4 * L) {
    p.kind = PH_HEAD;
    p.layer = L;
    p.units = 256 / 16;
    p.ksteps = d / 16;
    p.base = L * per_layer;
    p.w = m.whead;
    return p;
  }
  const LayerW lw = m.layers[p.layer];
  p.kind = ph % 4;
  switch (p.kind) {
    case PH_QKV:
      p.units = 3 * d / 16, p.ksteps = d / 16, p.w = lw.qkv;
      break;
    case PH_O:
      p.base += 3 * d / 16, p.units = d / 16, p.ksteps = d / 16, p.w = lw.o;
      break;
    case PH_W13:
      p.base += 4 * d / 16, p.units = 2 * F / 16, p.ksteps = d / 16, p.w = lw.w13;
      break;
    default:
      p.base += 4 * d / 16 + 2 * F / 16, p.units = d / 16, p.ksteps = F / 16, p.w = lw.w2;
      break;
  }
  return p;
}

__device__ __forceinline__ int first_unit(const Phase& p, int cta, int G) {
  return ((cta - p.base) % G + G) % G;
}

__device__ __forceinline__ unsigned epoch(const MegaArgs& m, int pass, int layer) {
  return m.epoch0 + (unsigned)(pass * (m.L + 1) + layer + 1);
}

// ---------------------------------------------------------------------------- producer
__device__ void mega_producer(const MegaArgs& m, unsigned char* ring, uint64_t* full, uint64_t* empty, int S, int lane) {
  const int G = gridDim.x, cta = blockIdx.x;
  const unsigned tile_bytes = 512u * m.planes;
  const uint64_t pol = l2_evict_first();
  unsigned it = 0;
  bool ok = true;
  for (int pass = 0; pass < m.max_passes && ok; ++pass) {
    if (pass > 0) {
      unsigned go = 0;
      if (lane == 0) {
        ok = wait_flag(m, m.flags + m.f_dec, epoch(m, pass - 1, m.L));
        go = ok ? __ldcg(m.dec_val) : 0u;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      go = __shfl_sync(0xffffffffu, go, 0);
      if (!ok || go == 0u) break;
    }
#pragma unroll 1
    for (int ph = 0; ph <= 4 * m.L && ok; ++ph) {
      const Phase p = phase_of(m, ph);
      const int nst = (p.ksteps + kStageTiles - 1) / kStageTiles;
#pragma unroll 1
      for (int u = first_unit(p, cta, G); u < p.units && ok; u += G) {
        const unsigned char* src = reinterpret_cast<const unsigned char*>(p.w) + (size_t)u * p.ksteps * tile_bytes;
#pragma unroll 1
        for (int st = 0; st < nst; ++st, ++it) {
          const int slot = it % S;
          const unsigned tiles = min(kStageTiles, p.ksteps - st * kStageTiles);
          if (lane == 0) {
            ok = wait_mbar(m, empty + slot, ((it / S) & 1) ^ 1);
            if (ok) {
              mbar_expect_tx(full + slot, tiles * tile_bytes);
              tma_1d(ring + (size_t)slot * kStageTiles * tile_bytes, src + (size_t)st * kStageTiles * tile_bytes, tiles * tile_bytes,
                     full + slot, pol);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
        }
      }
    }
  }
  // leave no copy in flight: every issued stage must have landed
  if (lane == 0) {
    const unsigned issued = it;
    const unsigned from = issued > (unsigned)S ? issued - S : 0;
#pragma unroll 1
    for (unsigned j = from; j < issued; ++j) {
      unsigned n = 0;
      while (!mbar_try(full + j % S, (j / S) & 1) && ++n < kSpinLimit) {
      }
    }
  }
}

// ---------------------------------------------------------------------------- consumer helpers
struct MegaSmem {
  unsigned char* ring;
  uint64_t* full;
  uint64_t* empty;
  int S;
  float* red;  // [8][16][16]
  float* ssr;  // [8][16]
  uint4* xs;   // phase input fragments [k-steps][NG][32 lanes] (shares space with the attention buffers)
  float* rsv;  // [16] RMS scale per row
  float* qs;
  float* ps;
  void* ks;
  void* vs;
  float* mrow;
  float* lrow;
  int* lim;
  int* plan_sh;
  int* misc;  // [0]: last-arrival flag, [1]: any-active
  int* rseq;  // this pass's row metadata, copied once per pass
  int* rpos;
  int* rlat;
  int* rbyte;
};

// Source rows of a phase input: value = a[k] (+ c[k] for the cross term).
struct XSrc {
  const float* a;
  const float* c;
};

// Input row of a phase (before the gain): QKV reads B_l = D_{l-1} + c_l (D_0 =
// embedding), O reads the attention output, W13 and the head read the
// residual stream, W2 reads the SwiGLU activations.
__device__ __forceinline__ XSrc x_src(const MegaArgs& m, const MegaSmem& sm, const Phase& p, int row) {
  XSrc x{nullptr, nullptr};
  const int d = m.d;
  if (p.kind == PH_QKV) {
    x.a = (p.layer == 0) ? m.ga.embed + (size_t)sm.rbyte[row] * d : m.h + (size_t)row * d;
    x.c = c_row(m.ga.c_lat, m.ga.max_lat, m.L, p.layer, d, sm.rseq[row], sm.rlat[row]);
  } else if (p.kind == PH_O) {
    x.a = m.att + (size_t)row * d;
  } else if (p.kind == PH_W2) {
    x.a = m.act + (size_t)row * m.F;
  } else {
    x.a = m.h + (size_t)row * d;
  }
  return x;
}
__device__ __forceinline__ float2 ld2(const float* p) { return __ldcg(reinterpret_cast<const float2*>(p)); }

// Flag of the i-th input that k-steps s0, s0 + 8, ... of phase p depend on:
// QKV and the head read the residual stream (W2 units), O reads attention
// heads (one per group), W13 the O units, W2 the W13 unit pairs.
__device__ __forceinline__ const unsigned* input_flag(const MegaArgs& m, const Phase& p, int s0, int n_groups, int i) {
  const unsigned* f = m.flags;
  switch (p.kind) {
    case PH_O: {
      const int spk = m.dh / 16;  // k-steps per head
      return f + m.f_att + (i % n_groups) * m.H + (s0 + 8 * (i / n_groups)) / spk;
    }
    case PH_W13:
      return f + m.f_o + s0 + 8 * i;
    case PH_W2:
      return f + m.f_w13 + 2 * (s0 + 8 * (i >> 1)) + (i & 1);
    default:  // QKV (layer > 0), head
      return f + m.f_w2 + s0 + 8 * i;
  }
}

// Wait (whole warp) until the inputs of k-steps s0, s0 + 8, ... (n of them)
// of phase p in this pass are written.  One polling loop for every phase
// kind keeps the kernel's code small.
__device__ __forceinline__ bool wait_inputs(const MegaArgs& m, const Phase& p, int pass, int s0, int n, int n_groups) {
  if (p.kind == PH_QKV && p.layer == 0) return true;
  int count = n;
  unsigned target = epoch(m, pass, p.layer);
  if (p.kind == PH_O) count = n * n_groups;
  else if (p.kind == PH_W2) count = 2 * n;
  else if (p.kind == PH_QKV) target = epoch(m, pass, p.layer - 1);
  else if (p.kind == PH_HEAD) target = epoch(m, pass, m.L - 1);
  return warp_wait(m, count, [&](int i) { return input_flag(m, p, s0, n_groups, i); }, target);
}

__device__ __forceinline__ const float* phase_gain(const MegaArgs& m, const Phase& p) {
  if (p.kind == PH_QKV) return m.layers[p.layer].attn_norm;
  if (p.kind == PH_W13) return m.layers[p.layer].ffn_norm;
  if (p.kind == PH_HEAD) return m.final_norm;
  return nullptr;
}

// Epilogue of one output pair, dispatched at run time so that one copy of the
// phase loop serves every projection (the kernel's code must stay small
// enough for the SM's instruction caches).
__device__ __forceinline__ void mega_epilogue(const GemmArgs& ga, int epi, int u, int r16, int row, float v0, float v1) {
  switch (epi) {
    case EPI_QKV:
      gemm_epilogue<EPI_QKV>(ga, u, r16, row, v0, v1);
      break;
    case EPI_XRESID:
      gemm_epilogue<EPI_XRESID>(ga, u, r16, row, v0, v1);
      break;
    case EPI_SWIGLU:
      gemm_epilogue<EPI_SWIGLU>(ga, u, r16, row, v0, v1);
      break;
    case EPI_RESID:
      gemm_epilogue<EPI_RESID>(ga, u, r16, row, v0, v1);
      break;
    default:
      gemm_epilogue<EPI_STORE>(ga, u, r16, row, v0, v1);
      break;
  }
}

// Phase input of this warp's k-steps warp, warp + 8, ... (nkw <= 8 of them) as
// split-bf16 B fragments in registers, and its lanes' sums of squares (the
// canonical order: per lane, k-steps in increasing order).  Every load is
// issued unconditionally (a dead row reads row 0, a k-step past the warp's
// share re-reads its last one; neither reaches an output) so all are in
// flight at once.  HASC: QKV input, which adds the cross term c_l.
template <int NG, bool HASC>
__device__ __forceinline__ void build_frags(const MegaArgs& m, const MegaSmem& sm, const Phase& p, int nr, int nkw,
                                            const float* gain, uint4 (&xf)[8][NG], float (&ss)[NG], int warp, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const bool norm = gain != nullptr;
  XSrc src[NG];
#pragma unroll
  for (int n = 0; n < NG; ++n) {
    ss[n] = 0.f;
    const int row = n * 8 + g;
    src[n] = x_src(m, sm, p, row < nr ? row : 0);
  }
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    if (half * 4 < nkw) {
      float2 ra[4][NG], rb[4][NG];
      float4 gv[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = min(half * 4 + jj, nkw - 1);
        const int k0 = (warp + 8 * j) * 16 + 2 * t;
#pragma unroll
        for (int n = 0; n < NG; ++n) {
          ra[jj][n] = ld2(src[n].a + k0);
          rb[jj][n] = ld2(src[n].a + k0 + 8);
          if constexpr (HASC) {
            const float2 c0 = ld2(src[n].c + k0), c8 = ld2(src[n].c + k0 + 8);
            ra[jj][n] = make_float2(ra[jj][n].x + c0.x, ra[jj][n].y + c0.y);
            rb[jj][n] = make_float2(rb[jj][n].x + c8.x, rb[jj][n].y + c8.y);
          }
        }
        gv[jj] = make_float4(1.f, 1.f, 1.f, 1.f);
        if (norm) gv[jj] = make_float4(__ldg(gain + k0), __ldg(gain + k0 + 1), __ldg(gain + k0 + 8), __ldg(gain + k0 + 9));
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = half * 4 + jj;
#pragma unroll
        for (int n = 0; n < NG; ++n) {
          const float2 a = ra[jj][n], b = rb[jj][n];
          if (norm && j < nkw) ss[n] = ss_add(ss[n], a.x, a.y, b.x, b.y);
          const XFrag f = make_xfrag(a.x * gv[jj].x, a.y * gv[jj].y, b.x * gv[jj].z, b.y * gv[jj].w);
          xf[j][n] = make_uint4(f.b0h, f.b1h, f.b0l, f.b1l);
        }
      }
    }
  }
}

// Phase with K <= 1024 (a unit is at most 8 / kTPW ring stages).  All eight warps
// work on every unit: warp w owns the k-steps s = w (mod 8) -- lane group w
// of the canonical order -- so it waits only for the inputs of its own
// k-steps and keeps their fragments in registers.  The CTA's units (up to
// kMegaUnits at a time) run together: one accumulator per unit per warp, so
// the units' MMA chains interleave; then one cross-warp reduction (the
// operation order of tile_reduce: warps in order, the RMS scale from the
// warps' sums of squares in order), one epilogue pass, one fence and the
// units' flags.
constexpr int kMegaUnits = 4;

template <int NG, int PL>
__device__ bool run_phase_units(const MegaArgs& m, const MegaSmem& sm, const Phase& p, int epi, int pass, unsigned& it, int nr,
                                int n_groups, const GemmArgs& ga, unsigned* flag_base, int tid) {
  constexpr int RB = 8 * NG;
  const int G = gridDim.x, cta = blockIdx.x;
  const int u0 = first_unit(p, cta, G);
  if (u0 >= p.units) return true;
  const int nunits = (p.units - u0 + G - 1) / G;
  const int nst = (p.ksteps + kStageTiles - 1) / kStageTiles;  // <= 8 / kTPW
  const unsigned it0 = it;
  it += (unsigned)(nunits * nst);
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const float* gain = phase_gain(m, p);
  const bool norm = gain != nullptr;
  const int nkw = (p.ksteps - warp + 7) / 8;  // k-steps of this warp (<= 8)
  trace_mark(m, pass, TR_PHASE_BEGIN << 8 | p.kind);
  bool ok = wait_inputs(m, p, pass, warp, nkw, n_groups);
  trace_mark(m, pass, TR_INPUTS << 8 | p.kind);
  uint4 xf[8][NG];
  float ss[NG];
  if (p.kind == PH_QKV) build_frags<NG, true>(m, sm, p, nr, nkw, gain, xf, ss, warp, lane);
  else build_frags<NG, false>(m, sm, p, nr, nkw, gain, xf, ss, warp, lane);
  if (norm) {
#pragma unroll
    for (int n = 0; n < NG; ++n) {
      float v = ss[n];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      if (t == 0) sm.ssr[warp * RB + n * 8 + g] = v;
    }
  }
  trace_mark(m, pass, TR_XLOADED << 8 | p.kind);
  const unsigned tile_bytes = 512u * PL;
  float* red = reinterpret_cast<float*>(sm.xs);  // [unit][warp][16][RB]
#pragma unroll 1
  for (int ug = 0; ug < nunits; ug += kMegaUnits) {
    const int nu = min(kMegaUnits, nunits - ug);
    float acc[kMegaUnits][NG][4];
#pragma unroll
    for (int jv = 0; jv < kMegaUnits; ++jv)
#pragma unroll
      for (int n = 0; n < NG; ++n) acc[jv][n][0] = acc[jv][n][1] = acc[jv][n][2] = acc[jv][n][3] = 0.f;
#pragma unroll
    for (int st = 0; st < 8 / kTPW; ++st) {
      if (st < nst) {
        const int ntiles = min(kStageTiles, p.ksteps - st * kStageTiles);
#pragma unroll
        for (int jv = 0; jv < kMegaUnits; ++jv) {
          if (jv < nu) {
            const unsigned itu = it0 + (unsigned)((ug + jv) * nst + st);
            const int slot = itu % sm.S;
            if (!wait_mbar(m, sm.full + slot, (itu / sm.S) & 1)) ok = false;
            const unsigned char* stage = sm.ring + (size_t)slot * kStageTiles * tile_bytes;
            uint4 w[kTPW][PL];
#pragma unroll
            for (int q = 0; q < kTPW; ++q)
#pragma unroll
              for (int pl = 0; pl < PL; ++pl)
                w[q][pl] = *reinterpret_cast<const uint4*>(stage + (size_t)min(8 * q + warp, ntiles - 1) * tile_bytes + pl * 512 + lane * 16);
#pragma unroll
            for (int q = 0; q < kTPW; ++q)
              if (8 * q + warp < ntiles)
#pragma unroll
                for (int n = 0; n < NG; ++n)
                  mma_step<PL>(acc[jv][n], w[q], XFrag{xf[st * kTPW + q][n].x, xf[st * kTPW + q][n].y, xf[st * kTPW + q][n].z, xf[st * kTPW + q][n].w});
            __syncwarp();
            if (lane == 0) mbar_arrive(sm.empty + slot);
          }
        }
      }
    }
#pragma unroll
    for (int jv = 0; jv < kMegaUnits; ++jv) {
      if (jv < nu) {
        float* rw = red + (size_t)(jv * 8 + warp) * 16 * RB;
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
      const float* ru = red + (size_t)jv * 8 * 16 * RB;
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
      mega_epilogue(ga, epi, u0 + (ug + jv) * G, r16, col, v0 * rs, v1 * rs);
    }
    consumer_sync();  // epilogue stores done, red free again
    if (tid == 0) {
      fence_acq_rel();
      for (int jv = 0; jv < nu; ++jv) st_relaxed(flag_base + u0 + (ug + jv) * G, epoch(m, pass, p.layer));
    }
    trace_mark(m, pass, TR_UNIT_DONE << 8 | p.kind);
  }
  return ok;
}

// Streamed-input phase (W2, K = F > 1024): inputs loaded stage by stage, one
// stage ahead.
template <int NG, int PL>
__device__ bool run_phase_streamed(const MegaArgs& m, const MegaSmem& sm, const Phase& p, int pass, unsigned& it, int nr,
                                   int n_groups, const GemmArgs& ga, unsigned* flag_base, int tid) {
  const int G = gridDim.x, cta = blockIdx.x;
  const int u0 = first_unit(p, cta, G);
  if (u0 >= p.units) return true;
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const unsigned tile_bytes = 512u * PL;
  const int nst = (p.ksteps + kStageTiles - 1) / kStageTiles;
  bool ok = true;
  trace_mark(m, pass, TR_PHASE_BEGIN << 8 | p.kind);
  ok = wait_inputs(m, p, pass, warp, (p.ksteps - warp + 7) / 8, n_groups);  // all of this warp's k-steps
  trace_mark(m, pass, TR_INPUTS << 8 | p.kind);
  XSrc src[NG];
#pragma unroll
  for (int n = 0; n < NG; ++n) src[n] = x_src(m, sm, p, n * 8 + g < nr ? n * 8 + g : 0);
  // unconditional loads (dead rows read row 0, k-steps past the end re-read
  // the last one; neither reaches an output) so all of a stage's are in flight together
  auto load = [&](int st, float2 (&xa)[kTPW][NG], float2 (&xb)[kTPW][NG]) {
#pragma unroll
    for (int jj = 0; jj < kTPW; ++jj) {
      const int ks = min(st * kStageTiles + 8 * jj + warp, p.ksteps - 1);
#pragma unroll
      for (int n = 0; n < NG; ++n) {
        xa[jj][n] = ld2(src[n].a + ks * 16 + 2 * t);
        xb[jj][n] = ld2(src[n].a + ks * 16 + 2 * t + 8);
      }
    }
    return ok;
  };
  // inputs prefetched D stages ahead in registers (an L2 round trip is much
  // longer than one stage's MMAs); stages run in groups of D so the register
  // ring is indexed at compile time
  constexpr int D = (kTPW == 4) ? 2 / NG : 1;
  for (int u = u0; u < p.units; u += G) {
    float acc[NG][4], ss[NG];
#pragma unroll
    for (int n = 0; n < NG; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = ss[n] = 0.f;
    float2 xa[D][kTPW][NG], xb[D][kTPW][NG];
#pragma unroll
    for (int d = 0; d < D; ++d)
      if (d < nst) ok = load(d, xa[d], xb[d]) && ok;
#pragma unroll 1
    for (int s0 = 0; s0 < nst; s0 += D) {
#pragma unroll
    for (int d = 0; d < D; ++d) {
      const int st = s0 + d;
      if (st < nst) {
        const int slot = it % sm.S;
        if (!wait_mbar(m, sm.full + slot, (it / sm.S) & 1)) ok = false;
        const unsigned char* stage = sm.ring + (size_t)slot * kStageTiles * tile_bytes;
        float2 (&ca)[kTPW][NG] = xa[d];
        float2 (&cb)[kTPW][NG] = xb[d];
        if ((st + 1) * kStageTiles <= p.ksteps) {  // full stage: weight loads first, then the chain
          uint4 w[kTPW][PL];
#pragma unroll
          for (int jj = 0; jj < kTPW; ++jj)
#pragma unroll
            for (int q = 0; q < PL; ++q)
              w[jj][q] = *reinterpret_cast<const uint4*>(stage + (size_t)(8 * jj + warp) * tile_bytes + q * 512 + lane * 16);
#pragma unroll
          for (int jj = 0; jj < kTPW; ++jj)
#pragma unroll
            for (int n = 0; n < NG; ++n) mma_step<PL>(acc[n], w[jj], make_xfrag(ca[jj][n].x, ca[jj][n].y, cb[jj][n].x, cb[jj][n].y));
        } else {
#pragma unroll
          for (int jj = 0; jj < kTPW; ++jj) {
            const int tile = 8 * jj + warp;
            if (st * kStageTiles + tile < p.ksteps) {
              uint4 w[PL];
#pragma unroll
              for (int q = 0; q < PL; ++q) w[q] = *reinterpret_cast<const uint4*>(stage + (size_t)tile * tile_bytes + q * 512 + lane * 16);
#pragma unroll
              for (int n = 0; n < NG; ++n) mma_step<PL>(acc[n], w, make_xfrag(ca[jj][n].x, ca[jj][n].y, cb[jj][n].x, cb[jj][n].y));
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sm.empty + slot);
        ++it;
        if (st + D < nst) ok = load(st + D, xa[d], xb[d]) && ok;
      }
    }
    }
    trace_mark(m, pass, TR_KLOOP << 8 | p.kind);
    tile_reduce<NG>(acc, ss, false, sm.red, sm.ssr, nr, p.ksteps * 16, m.eps, tid, 256, consumer_sync,
                    [&](int r16, int col, float v0, float v1) { mega_epilogue(ga, EPI_RESID, u, r16, col, v0, v1); });
    trace_mark(m, pass, TR_REDUCED << 8 | p.kind);
    consumer_sync();
    if (tid == 0) st_release(flag_base + u, epoch(m, pass, p.layer));
    trace_mark(m, pass, TR_UNIT_DONE << 8 | p.kind);
  }
  return ok;
}

// Attention of layer l: items (group, head, chunk) dealt round-robin; the
// last CTA to finish a (group, head) combines its chunks and raises the flag.
template <int DH, typename KVT>
__device__ bool run_attention(const MegaArgs& m, const MegaSmem& sm, int layer, int pass, int n_groups, int tid) {
  const int G = gridDim.x, cta = blockIdx.x;
  AttnArgs a = m.aa;
  a.layer = layer;
  const int tph = DH / 16;
  const int tiles_sec = m.d / 16;
  int total = 0;
  for (int g = 0; g < n_groups; ++g) total += m.H * ((__ldcg(m.rows.g_kmax + g) + a.CH - 1) / a.CH);
  bool ok = true;
  KVT* ks = static_cast<KVT*>(sm.ks);
  KVT* vs = static_cast<KVT*>(sm.vs);
  for (int item = cta; item < total; item += G) {
    int g = 0, rem = item, nch = 0;
    for (; g < n_groups; ++g) {
      nch = (__ldcg(m.rows.g_kmax + g) + a.CH - 1) / a.CH;
      if (rem < m.H * nch) break;
      rem -= m.H * nch;
    }
    const int h = rem / nch, c = rem % nch;
    const int seq = __ldcg(m.rows.g_seq + g), kmax = __ldcg(m.rows.g_kmax + g), fresh = __ldcg(m.rows.g_fresh + g);
    const int t0 = c * a.CH, t1 = min(t0 + a.CH, kmax);
    trace_mark(m, pass, TR_ATT_BEGIN << 8);
    // keys cached before this pass can be fetched before q/k/v of this pass exist
    attn_load_kv<DH, KVT>(a, seq, h, t0, t0, min(t1, fresh), ks, vs, tid, 256);
    cp_async_commit();
    if (tid < 32)
      ok = warp_wait(m, 3 * tph, [&](int i) { return m.flags + m.f_qkv + (i / tph) * tiles_sec + h * tph + i % tph; },
                     epoch(m, pass, layer)) && ok;
    consumer_sync();
    trace_mark(m, pass, TR_ATT_QKV << 8);
    attn_load_kv<DH, KVT>(a, seq, h, t0, max(t0, fresh), t1, ks, vs, tid, 256);
    cp_async_commit();
    cp_async_wait<0>();
    consumer_sync();
    trace_mark(m, pass, TR_ATT_LOADED << 8);
    attn_partial_compute<DH, KVT, decltype(&consumer_sync)>(
        a, g, h, c, sm.qs, sm.ps, ks, vs, sm.mrow, sm.lrow, sm.lim, tid, 256, consumer_sync,
        [&](int step) { trace_mark(m, pass, TR_ATT_STEP << 8 | step); });
    consumer_sync();
    trace_mark(m, pass, TR_ATT_COMPUTED << 8);
    if (tid == 0) {
      __threadfence();
      const unsigned old = atomicAdd(m.attn_cnt + g * m.H + h, 1u);
      sm.misc[0] = (old == (unsigned)(nch - 1));
      __threadfence();
    }
    consumer_sync();
    if (sm.misc[0]) {
      const int row0 = __ldcg(m.rows.g_row0 + g), nr = __ldcg(m.rows.g_nrows + g);
      for (int r = tid >> 5; r < nr; r += 8) attn_combine_row<DH>(a, row0 + r, h, tid & 31);
      consumer_sync();
      if (tid == 0) {
        m.attn_cnt[g * m.H + h] = 0u;
        st_release(m.flags + m.f_att + g * m.H + h, epoch(m, pass, layer));
      }
    }
    consumer_sync();
    trace_mark(m, pass, TR_ATT_DONE << 8 | sm.misc[0]);
  }
  return ok;
}

// After the head of pass `pass`: statistics, the mode's bookkeeping, the
// decision to go on, the plan of the next pass (CTA 0 only).
__device__ void mega_bookkeeping(const MegaArgs& m, const MegaSmem& sm, int pass, int nr, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  if (tid < 32) warp_wait(m, 16, [&](int u) { return m.flags + m.f_head + u; }, epoch(m, pass, m.L));
  if (tid == 0) sm.misc[1] = 0;
  consumer_sync();
  for (int r = warp; r < nr; r += 8) {
    float c, g, e;
    int p;
    head_stats_row(m.logits + (size_t)r * 256, lane, c, p, g, e);
    if (lane == 0) {
      m.conf[r] = c;
      m.pred[r] = p;
      m.gap[r] = g;
      m.ent[r] = e;
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
  if (cont) {
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
    *(volatile unsigned*)m.dec_val = cont ? 1u : 0u;
    __threadfence();
    st_release(m.flags + m.f_dec, epoch(m, pass, m.L));
  }
}

template <int NG, int PL, int DH, typename KVT>
__global__ void __launch_bounds__(kMegaThreads, 1) k_mega(MegaArgs m) {
  extern __shared__ __align__(1024) unsigned char mega_smem[];
  __shared__ uint64_t bars[2 * 16];
  __shared__ int plan_sh[3 * (kMaxCallBatch + 1)];
  __shared__ int misc[4];
  __shared__ float mrow[kAttnRows], lrow[kAttnRows];
  __shared__ int lim[kAttnRows];
  __shared__ int rmeta[4][8 * kMegaMaxNG];
  __shared__ int rpage[8 * kMegaMaxNG];                       // KV page of each row's position
  __shared__ float rope_c[8 * kMegaMaxNG * 32], rope_s[8 * kMegaMaxNG * 32];  // [row][dh/2], dh <= 64

  const unsigned tile_bytes = 512u * PL;
  const unsigned slot_bytes = kStageTiles * tile_bytes;
  MegaSmem sm;
  sm.S = min(16, (int)(kRingBytes / slot_bytes));
  sm.ring = mega_smem;
  unsigned char* p = mega_smem + kRingBytes;
  sm.red = reinterpret_cast<float*>(p);
  p += 8 * 16 * 8 * kMegaMaxNG * 4;
  sm.ssr = reinterpret_cast<float*>(p);
  p += 8 * 8 * kMegaMaxNG * 4;
  sm.rsv = reinterpret_cast<float*>(p);
  p += 16 * 4;
  sm.xs = reinterpret_cast<uint4*>(p);  // the phases' reduction buffer shares space with the attention buffers
  sm.qs = reinterpret_cast<float*>(p);
  p += kAttnRows * DH * 4;
  sm.ps = reinterpret_cast<float*>(p);
  p += kAttnRows * m.aa.CH * 4;
  sm.ks = p;
  p += m.aa.CH * kv_stride<DH, KVT>() * sizeof(KVT);
  sm.vs = p;
  sm.full = bars;
  sm.empty = bars + 16;
  sm.mrow = mrow;
  sm.lrow = lrow;
  sm.lim = lim;
  sm.plan_sh = plan_sh;
  sm.misc = misc;
  sm.rseq = rmeta[0];
  sm.rpos = rmeta[1];
  sm.rlat = rmeta[2];
  sm.rbyte = rmeta[3];

  const int tid = threadIdx.x;
  if (tid == 0) {
    s_trace_n = 0;
    for (int i = 0; i < sm.S; ++i) {
      mbar_init(sm.full + i, 1);
      mbar_init(sm.empty + i, kMegaConsumers);
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();

  if (tid >= 256) {  // producer warp
    mega_producer(m, sm.ring, sm.full, sm.empty, sm.S, tid & 31);
    return;
  }
  unsigned it = 0;
  bool ok = true;
  for (int pass = 0; pass < m.max_passes && ok; ++pass) {
    if (pass > 0) {
      if (tid == 0) misc[2] = wait_flag(m, m.flags + m.f_dec, epoch(m, pass - 1, m.L)) ? (int)__ldcg(m.dec_val) : -1;
      consumer_sync();
      const int go = misc[2];
      consumer_sync();
      if (go <= 0) {
        ok = go == 0;
        break;
      }
    }
    const int nr = __ldcg(m.rows.n_rows);
    const int n_groups = __ldcg(m.rows.n_groups);
    if (tid < 8 * kMegaMaxNG) {  // rows past nr get harmless in-range values (inputs are loaded unconditionally)
      const bool live = tid < nr;
      sm.rseq[tid] = live ? __ldcg(m.rows.seq + tid) : 0;
      sm.rpos[tid] = live ? __ldcg(m.rows.pos + tid) : 0;
      sm.rlat[tid] = live ? __ldcg(m.rows.lat + tid) : 0;
      sm.rbyte[tid] = live ? __ldcg(m.rows.byte + tid) : 0;
    }
    consumer_sync();
    {  // this pass's rotary factors and KV pages per row (dead rows: position 0)
      const int half = m.dh / 2;
      for (int i = tid; i < 8 * kMegaMaxNG * half; i += 256) {
        const size_t src = (size_t)sm.rpos[i / half] * half + i % half;
        rope_c[i] = __ldg(m.ga.rope_cos + src);
        rope_s[i] = __ldg(m.ga.rope_sin + src);
      }
      if (tid < 8 * kMegaMaxNG) {
        const int pi = sm.rpos[tid] / m.ga.PT;
        rpage[tid] = (pi < m.ga.max_pages) ? __ldcg(m.ga.page_table + sm.rseq[tid] * m.ga.max_pages + pi) : -1;
      }
    }
    consumer_sync();
    trace_mark(m, pass, TR_PASS << 8);
    // Steps of a pass: per layer QKV, attention, O, W13, W2; then the byte
    // head.  One call site per routine keeps a single copy of each in the
    // kernel, small enough for the SM's instruction caches.
    GemmArgs ga = m.ga;
    ga.row_seq = sm.rseq;
    ga.row_pos = sm.rpos;
    ga.row_lat = sm.rlat;
    ga.row_byte = sm.rbyte;
    ga.rope_cos = rope_c;
    ga.rope_sin = rope_s;
    ga.rope_by_row = 1;
    ga.row_page = rpage;
    for (int step = 0; step <= 5 * m.L && ok; ++step) {
      const int l = step / 5, k = step - 5 * l;
      if (k == 1) {
        ok = run_attention<DH, KVT>(m, sm, l, pass, n_groups, tid) && ok;
        continue;
      }
      const bool head = l == m.L;
      const Phase p = phase_of(m, head ? 4 * m.L : 4 * l + (k == 0 ? 0 : k - 1));
      ga.layer = head ? 0 : l;
      int epi = EPI_STORE;
      unsigned* fb = m.flags + m.f_head;
      if (head) {
        ga.out = m.logits, ga.ldo = 256;
      } else if (k == 0) {
        epi = EPI_QKV, fb = m.flags + m.f_qkv;
      } else if (k == 2) {
        epi = EPI_XRESID, fb = m.flags + m.f_o, ga.out = m.h, ga.ldo = m.d;
      } else if (k == 3) {
        epi = EPI_SWIGLU, fb = m.flags + m.f_w13, ga.out = m.act, ga.ldo = m.F;
      } else {
        epi = EPI_RESID, fb = m.flags + m.f_w2, ga.out = m.h, ga.ldo = m.d;
      }
      if (k == 4 && !head && p.ksteps > 64) ok = run_phase_streamed<NG, PL>(m, sm, p, pass, it, nr, n_groups, ga, fb, tid) && ok;
      else ok = run_phase_units<NG, PL>(m, sm, p, epi, pass, it, nr, n_groups, ga, fb, tid) && ok;
    }
    if (!ok) break;
    trace_mark(m, pass, TR_HEAD << 8);
    if (blockIdx.x == 0 && ok) mega_bookkeeping(m, sm, pass, nr, tid);
    trace_mark(m, pass, TR_BOOK << 8);
  }
}

}  // namespace bltdec
