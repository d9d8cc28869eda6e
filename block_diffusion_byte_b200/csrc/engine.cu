// Host side of the Fast-BLT local-decoder engine: weight layout, paged KV
// pool, latent cache, per-call sequencing of decoder passes, and the C ABI of
// bltdec.h.  Every decoder step runs in the kernels of kernels.cuh.
#include <algorithm>
#include <mutex>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "bltdec.h"
#include "kernels.cuh"
#include "mega.cuh"
#include "tc_gemm.cuh"
#include "sampling.cuh"

using namespace bltdec;

namespace {

// NVTX range for the lifetime of a scope (per C-ABI call, per decoder pass);
// free unless a profiler is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

struct Mat {
  uint4* w = nullptr;
  int N = 0, K = 0, planes = 1;
  // BLT_FLAG_TENSOR_CORES: the same rows (same order), row-major bf16, and its TMA map (box 64 x tc_bn)
  __nv_bfloat16* wr = nullptr;
  int tc_bn = 0;
  CUtensorMap tmap{};
  size_t bytes() const { return (size_t)N * K * 2 * planes; }
};

uint16_t bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  u = u + 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
float bf16_to_f(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

}  // namespace

struct blt_dec {
  blt_dec_config cfg{};
  cudaStream_t stream = nullptr;
  bool own_stream = false;
  int L = 0, d = 0, H = 0, dh = 0, F = 0, dg = 0, V = 0, planes = 1;
  int PT = 0, max_pages = 0, n_pages = 0, CH = 0, CMAX = 0;
  std::vector<Mat> qkv, o, w13, w2;
  Mat vc_all, oc_all;  // latent projections of all layers, stacked along N (layer l: tiles l*d/16 ..)
  int proj_rows = 0;   // latents per projection chunk (tmp holds proj_rows x L*d)
  std::vector<float*> attn_norm, ffn_norm;
  Mat head;
  float* embed = nullptr;
  float* final_norm = nullptr;
  float *rope_cos = nullptr, *rope_sin = nullptr;
  void* kv = nullptr;  // KV pool, element type per kv_f32
  int kv_f32 = 0;
  int* page_table = nullptr;
  std::vector<int> pt_host, free_pages, seq_npages;
  float* c_lat = nullptr;
  float *h = nullptr, *rs = nullptr, *q = nullptr, *att = nullptr, *act = nullptr, *logits = nullptr, *tmp = nullptr;
  float2* part_ml = nullptr;
  float* part_o = nullptr;
  float *conf = nullptr, *gap = nullptr;
  int* pred = nullptr;
  RowsDev rows{};
  int *lat_seq = nullptr, *lat_slot = nullptr, *n_lat_rows = nullptr;
  SeqDev sd{};
  std::vector<void*> allocs;
  int state = 0;  // 0 ready, 1 draft waiting
  int draft_k = 0, draft_batch = 0;
  bool draft_sampled = false;  // the waiting draft was drawn (its distributions are in sa.qdist)
  std::vector<int> kv_ub, nlat_ub;
  int* mirror = nullptr;  // pinned [2*max_batch]: kv_len, n_lat
  cudaEvent_t mirror_ev = nullptr;
  bool mirror_pending = false;
  std::string err;
  unsigned long long weight_bytes_per_pass = 0, kv_bytes_per_key = 0;
  unsigned long long launches = 0;  // kernels launched (host count)
  unsigned long long persistent_calls = 0;  // calls served by the persistent kernel
  int eb = 0;             // the running call unmasks by EB sampling (blt_dec_diffuse_block_eb)
  float* ent = nullptr;   // per-row entropy of the byte head
  // pass timing (BLT_FLAG_TIME_PASSES): event pairs recorded around passes
  std::vector<cudaEvent_t> tev;
  size_t tev_used = 0;
  unsigned long long timed_passes = 0, pass_ns = 0;
  // persistent pass kernel
  bool mega_ok = false;
  int nsm = 0;
  LayerW* d_layers = nullptr;
  unsigned* flags = nullptr;  // [0] decision epoch, [1] pass-end arrivals
  unsigned* dec_val = nullptr;
  int* abort_flag = nullptr;  // flags + 2: reset with the pass-end arrivals in one memset
  unsigned long long calls = 0;  // engine calls served (counted on the host)
  unsigned epoch = 0;
  unsigned long long* xbuf = nullptr;  // exchange words of the persistent kernel (one allocation)
  size_t xbuf_words = 0;
  unsigned long long *x_h = nullptr, *x_q = nullptr, *x_k = nullptr, *x_v = nullptr, *x_att = nullptr, *x_act = nullptr,
                     *x_w2p = nullptr, *x_logit = nullptr, *x_part = nullptr;
  int x_cmax = 0;
  // tcgen05 GEMM (BLT_FLAG_TENSOR_CORES): prepared activation planes [RL][max(d, F)] and row scales
  bool tc = false;
  // split-K of small GEMV grids over K segments (W2 of small passes): workspace [nseg][seg_rows][seg_n]
  float* seg_ws = nullptr;
  int seg_rows = 0, seg_n = 0, seg_nmax = 0, sm_count = 0;
  __nv_bfloat16 *tc_hi = nullptr, *tc_lo = nullptr;
  float* tc_rs = nullptr;
  CUtensorMap tc_hi_d{}, tc_lo_d{}, tc_hi_f{}, tc_lo_f{};  // views with row stride d and F
  unsigned long long tc_gemms = 0;
  // stochastic decoding (the *_sampled entry points): on for the duration of such a call
  bool samp_on = false;
  SampleArgs sa{};
  // persistent kernel: sleep between polls of a wait (ns; first 32 polls, then the rest).
  // Tuning knob: BLTDEC_SPIN_NS="<first>,<rest>".
  unsigned spin_ns[2] = {32, 128};
  // attention items per SM up to which a small pass runs in the persistent kernel.
  // Tuning knob: BLTDEC_MEGA_ITEMS_PER_SM=<n>.
  int mega_items_per_sm = 8;
  // debug: BLTDEC_TRACE=<file> appends device timestamps of each persistent launch's first pass
  unsigned long long* trace = nullptr;
  std::string trace_path;
  int trace_pending = 0;
  // blt_dec_upload: a ring of pinned bounce buffers, each reused once its last copy has run
  struct Bounce {
    void* p = nullptr;
    size_t cap = 0;
    cudaEvent_t done = nullptr;
  };
  static constexpr int kUpSlots = 4;
  static constexpr size_t kUpSmall = 256 * 1024;  // ring buffers' size; larger copies use up_large
  Bounce up[kUpSlots];
  int up_next = 0;
  Bounce up_large;  // grows to the largest copy seen (prefill rows and latents)
  Bounce down;      // blt_dec_download
};

namespace {

int fail(blt_dec* h, int code, const char* fmt, ...) __attribute__((format(printf, 3, 4)));
int fail(blt_dec* h, int code, const char* fmt, ...) {
  if (h) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    h->err = buf;
  }
  return code;
}

#define CK(call)                                                                                     \
  do {                                                                                               \
    cudaError_t e_ = (call);                                                                         \
    if (e_ != cudaSuccess) return fail(h, BLT_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_));   \
  } while (0)

template <class T>
int dalloc(blt_dec* h, T** p, size_t count) {
  void* v = nullptr;
  cudaError_t e = cudaMalloc(&v, std::max<size_t>(count, 1) * sizeof(T));
  if (e != cudaSuccess) return fail(h, BLT_ERR_CUDA, "cudaMalloc(%zu): %s", count * sizeof(T), cudaGetErrorString(e));
  h->allocs.push_back(v);
  *p = static_cast<T*>(v);
  return BLT_OK;
}

#define TRY(x)                  \
  do {                          \
    int r_ = (x);               \
    if (r_ != BLT_OK) return r_; \
  } while (0)

// Pack W (rows given by src_row(tile_row) of a [*, K] fp32 matrix) into
// m16k16 tensor-core A-fragment order: tile (mt, ks), plane p, lane l holds
// rows g, g+8 and columns 2t, 2t+1, 2t+8, 2t+9 (g = l/4, t = l%4).
// TMA map of a row-major bf16 matrix [outer][inner]: boxes of 64 inner elements
// (one 128-byte swizzle atom) x box_outer rows, zero fill outside.
typedef CUresult (*TensorMapEncodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                         const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                         CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
int tc_map(blt_dec* h, CUtensorMap* map, const void* base, int inner, int outer, int box_outer) {
  static TensorMapEncodeTiled encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    CK(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
    if (!fn || q != cudaDriverEntryPointSuccess) return fail(h, BLT_ERR_CUDA, "cuTensorMapEncodeTiled not available");
    encode = reinterpret_cast<TensorMapEncodeTiled>(fn);
  }
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  const cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kTcBK, (cuuint32_t)box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(h, BLT_ERR_CUDA, "cuTensorMapEncodeTiled: error %d", (int)r);
  return BLT_OK;
}

template <class RowFn>
int pack_matrix(blt_dec* h, Mat& m, int N, int K, int planes, RowFn src_row, bool tc_copy = false) {
  m.N = N;
  m.K = K;
  m.planes = planes;
  const int ntm = N / 16, nks = K / 16;
  std::vector<uint16_t> buf((size_t)N * K * planes);
  for (int mt = 0; mt < ntm; ++mt) {
    const float* ra[8];
    const float* rb[8];
    for (int g = 0; g < 8; ++g) {
      ra[g] = src_row(mt * 16 + g);
      rb[g] = src_row(mt * 16 + g + 8);
    }
    for (int ks = 0; ks < nks; ++ks) {
      uint16_t* tile = buf.data() + ((size_t)mt * nks + ks) * planes * 256;
      for (int lane = 0; lane < 32; ++lane) {
        const int g = lane >> 2, t = lane & 3, c = ks * 16 + 2 * t;
        const float v[8] = {ra[g][c], ra[g][c + 1], rb[g][c], rb[g][c + 1], ra[g][c + 8], ra[g][c + 9], rb[g][c + 8], rb[g][c + 9]};
        for (int e = 0; e < 8; ++e) {
          const uint16_t hi = bf16_rne(v[e]);
          tile[lane * 8 + e] = hi;
          if (planes == 2) tile[256 + lane * 8 + e] = bf16_rne(v[e] - bf16_to_f(hi));
        }
      }
    }
  }
  TRY(dalloc(h, &m.w, buf.size() * 2 / 16));
  CK(cudaMemcpy(m.w, buf.data(), buf.size() * 2, cudaMemcpyHostToDevice));
  if (tc_copy && h->tc && planes == 1 && K % kTcBK == 0) {
    std::vector<uint16_t> rm((size_t)N * K);
    for (int r = 0; r < N; ++r) {
      const float* src = src_row(r);
      for (int k = 0; k < K; ++k) rm[(size_t)r * K + k] = bf16_rne(src[k]);
    }
    m.tc_bn = N >= 2048 ? 128 : N >= 512 ? 64 : 32;
    if (N % m.tc_bn) return BLT_OK;  // stays on the GEMV path
    TRY(dalloc(h, &m.wr, rm.size()));
    CK(cudaMemcpy(m.wr, rm.data(), rm.size() * 2, cudaMemcpyHostToDevice));
    TRY(tc_map(h, &m.tmap, m.wr, K, N, m.tc_bn));
  }
  return BLT_OK;
}

int upload(blt_dec* h, float** dst, const float* src, size_t n) {
  TRY(dalloc(h, dst, n));
  CK(cudaMemcpy(*dst, src, n * 4, cudaMemcpyHostToDevice));
  return BLT_OK;
}

// ---------------------------------------------------------------------------- pass timing
int pass_begin(blt_dec* h) {
  if (!(h->cfg.flags & BLT_FLAG_TIME_PASSES)) return BLT_OK;
  if (h->tev_used + 2 > h->tev.size()) {
    for (int i = 0; i < 64; ++i) {
      cudaEvent_t e;
      CK(cudaEventCreate(&e));
      h->tev.push_back(e);
    }
  }
  CK(cudaEventRecord(h->tev[h->tev_used], h->stream));
  return BLT_OK;
}
int pass_end(blt_dec* h) {
  if (!(h->cfg.flags & BLT_FLAG_TIME_PASSES)) return BLT_OK;
  CK(cudaEventRecord(h->tev[h->tev_used + 1], h->stream));
  h->tev_used += 2;
  return BLT_OK;
}
// Fold recorded pass times into the counters (the stream must be idle).
int drain_timing(blt_dec* h) {
  for (size_t i = 0; i + 1 < h->tev_used; i += 2) {
    float ms = 0.f;
    CK(cudaEventElapsedTime(&ms, h->tev[i], h->tev[i + 1]));
    h->pass_ns += (unsigned long long)(ms * 1e6);
  }
  h->tev_used = 0;
  return BLT_OK;
}

// ---------------------------------------------------------------------------- GEMM launch
template <int NG, int PL, int EPI>
constexpr int gemm_stages() {
  return NG >= 8 ? 3 : 4;
}
template <int NG, int PL, int EPI>
size_t gemm_smem() {
  constexpr int RB = 8 * NG;
  // activation stages, the RMS partials [8][RB], and the K-segment fold buffer [8][16][RB]
  return (size_t)gemm_stages<NG, PL, EPI>() * RB * kXStride * 4 + 8 * RB * 4 + 8 * 16 * RB * 4;
}

template <int NG, int PL, int EPI>
int set_gemm_attr(blt_dec* h) {
  CK(cudaFuncSetAttribute(k_gemm<NG, PL, EPI, gemm_stages<NG, PL, EPI>()>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                          (int)gemm_smem<NG, PL, EPI>()));
  return BLT_OK;
}

template <int EPI>
int set_tc_attrs(blt_dec* h) {
  CK(cudaFuncSetAttribute(k_tc_gemm<32, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc_smem_bytes(32)));
  CK(cudaFuncSetAttribute(k_tc_gemm<64, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc_smem_bytes(64)));
  CK(cudaFuncSetAttribute(k_tc_gemm<128, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc_smem_bytes(128)));
  return BLT_OK;
}

template <int EPI>
int set_attrs_epi(blt_dec* h) {
  TRY((set_gemm_attr<1, 1, EPI>(h)));
  TRY((set_gemm_attr<2, 1, EPI>(h)));
  TRY((set_gemm_attr<4, 1, EPI>(h)));
  TRY((set_gemm_attr<8, 1, EPI>(h)));
  TRY((set_gemm_attr<1, 2, EPI>(h)));
  TRY((set_gemm_attr<2, 2, EPI>(h)));
  TRY((set_gemm_attr<4, 2, EPI>(h)));
  TRY((set_gemm_attr<8, 2, EPI>(h)));
  return BLT_OK;
}

template <int NG, int PL, int EPI>
void launch_ng(blt_dec* h, const GemmArgs& a, int rows_ub) {
  constexpr int RB = 8 * NG;
  dim3 grid(a.N / 16, (rows_ub + RB - 1) / RB, a.seg_ws ? a.K / kSegCols : 1);
  k_gemm<NG, PL, EPI, gemm_stages<NG, PL, EPI>()><<<grid, kThreads, gemm_smem<NG, PL, EPI>(), h->stream>>>(a);
}

template <int BN, int EPI>
void launch_tc(blt_dec* h, const Mat& m, const GemmArgs& a, int rows_ub) {
  const bool kd = m.K == h->d;
  dim3 grid(m.N / BN, (rows_ub + kTcBM - 1) / kTcBM);
  k_tc_gemm<BN, EPI><<<grid, 128, tc_smem_bytes(BN), h->stream>>>(kd ? h->tc_hi_d : h->tc_hi_f, kd ? h->tc_lo_d : h->tc_lo_f,
                                                                  m.tmap, a, h->tc_rs, 500000000ull);
}

// The projection on the tcgen05 GEMM: activation prep, then the tiles.
template <int EPI>
int tc_gemm(blt_dec* h, const Mat& m, GemmArgs a, int rows_ub) {
  a.w = nullptr;
  a.N = m.N;
  a.K = m.K;
  a.status = h->sd.status;
  k_tc_prep<<<rows_ub, 256, 0, h->stream>>>(a.X, a.ldx, m.K, a.gain, a.eps, a.n_rows, rows_ub, h->tc_hi, h->tc_lo, h->tc_rs);
  if (m.tc_bn == 128) launch_tc<128, EPI>(h, m, a, rows_ub);
  else if (m.tc_bn == 64) launch_tc<64, EPI>(h, m, a, rows_ub);
  else launch_tc<32, EPI>(h, m, a, rows_ub);
  h->launches += 2;
  h->tc_gemms += 1;
  CK(cudaGetLastError());
  return BLT_OK;
}

template <int EPI>
int gemm(blt_dec* h, const Mat& m, GemmArgs a, int rows_ub) {
  if (rows_ub <= 0) return BLT_OK;
  if constexpr (EPI == EPI_STORE || EPI == EPI_RESID || EPI == EPI_SWIGLU || EPI == EPI_QKV) {
    if (h->tc && rows_ub >= kTcMinRows && m.wr) return tc_gemm<EPI>(h, m, a, rows_ub);
  }
  a.w = m.w;
  a.N = m.N;
  a.K = m.K;
  a.status = h->sd.status;
  const int ng = rows_ub <= 8 ? 1 : rows_ub <= 16 ? 2 : rows_ub <= 32 ? 4 : 8;
  h->launches += 1;
  // A grid of fewer CTAs than half the SMs with K in several canonical segments (W2 of a small
  // pass): one CTA per (tile, segment), then k_seg_finish adds the segment sums in order --
  // the same additions in the same order as one CTA folding them, so the same bits.
  const int nseg = m.K / kSegCols;
  const long long tiles = (long long)(m.N / 16) * ((rows_ub + 8 * ng - 1) / (8 * ng));
  const bool split = h->seg_ws && a.gain == nullptr && m.K > kSegCols && m.K % kSegCols == 0 && nseg <= h->seg_nmax &&
                     m.N <= h->seg_n && rows_ub <= h->seg_rows && 2 * tiles <= h->sm_count;
  if (split) {
    a.seg_ws = h->seg_ws;
    a.seg_rows = h->seg_rows;
  }
  if (m.planes == 1) {
    if (ng == 1) launch_ng<1, 1, EPI>(h, a, rows_ub);
    else if (ng == 2) launch_ng<2, 1, EPI>(h, a, rows_ub);
    else if (ng == 4) launch_ng<4, 1, EPI>(h, a, rows_ub);
    else launch_ng<8, 1, EPI>(h, a, rows_ub);
  } else {
    if (ng == 1) launch_ng<1, 2, EPI>(h, a, rows_ub);
    else if (ng == 2) launch_ng<2, 2, EPI>(h, a, rows_ub);
    else if (ng == 4) launch_ng<4, 2, EPI>(h, a, rows_ub);
    else launch_ng<8, 2, EPI>(h, a, rows_ub);
  }
  if (split) {
    const long long pairs = (long long)rows_ub * (m.N / 2);
    k_seg_finish<EPI><<<(unsigned)((pairs + 255) / 256), 256, 0, h->stream>>>(a, nseg);
    h->launches += 1;
  }
  CK(cudaGetLastError());
  return BLT_OK;
}

GemmArgs base_args(blt_dec* h) {
  GemmArgs a{};
  a.n_rows = h->rows.n_rows;
  a.kv = h->kv;
  a.kv_f32 = h->kv_f32;
  a.page_table = h->page_table;
  a.max_pages = h->max_pages;
  a.PT = h->PT;
  a.L = h->L;
  a.H = h->H;
  a.dh = h->dh;
  a.d = h->d;
  a.row_seq = h->rows.seq;
  a.row_pos = h->rows.pos;
  a.row_lat = h->rows.lat;
  a.row_byte = h->rows.byte;
  a.embed = h->embed;
  a.c_lat = h->c_lat;
  a.eps = h->cfg.norm_eps;
  a.rope_cos = h->rope_cos;
  a.rope_sin = h->rope_sin;
  a.max_lat = h->cfg.max_latents;
  a.status = h->sd.status;
  return a;
}

// Shared memory of k_attn_partial for groups of at most `rows` rows.
size_t attn_smem_bytes(const blt_dec* h, int rows = kAttnRows) {
  const int es = h->kv_f32 ? 4 : 2;
  return (size_t)(rows * h->dh + rows * h->CH) * 4 + (size_t)2 * h->CH * (h->dh + 16 / es) * es;
}
AttnArgs attn_args(blt_dec* h) {
  AttnArgs aa{};
  aa.kv = h->kv;
  aa.page_table = h->page_table;
  aa.max_pages = h->max_pages;
  aa.PT = h->PT;
  aa.L = h->L;
  aa.H = h->H;
  aa.dh = h->dh;
  aa.d = h->d;
  aa.rows = h->rows;
  aa.CH = h->CH;
  aa.CMAX = h->CMAX;
  aa.scale = 1.0f / std::sqrt((float)h->dh);
  aa.q = h->q;
  aa.part_ml = h->part_ml;
  aa.part_o = h->part_o;
  aa.att = h->att;
  aa.status = h->sd.status;
  return aa;
}
template <typename KVT, int ROWS>
void launch_attn_r(blt_dec* h, dim3 ag, const AttnArgs& aa) {
  const size_t smem = attn_smem_bytes(h, ROWS);
  if (h->dh == 64) k_attn_partial<64, KVT, ROWS><<<ag, 128, smem, h->stream>>>(aa);
  else if (h->dh == 32) k_attn_partial<32, KVT, ROWS><<<ag, 128, smem, h->stream>>>(aa);
  else if (h->dh == 128) k_attn_partial<128, KVT, ROWS><<<ag, 128, smem, h->stream>>>(aa);
  else k_attn_partial<16, KVT, ROWS><<<ag, 128, smem, h->stream>>>(aa);
}
// grp_rows_ub: the most rows any attention group of the pass can hold; a smaller bound
// selects a variant with less shared memory, so more blocks share an SM.
template <typename KVT>
void launch_attn_t(blt_dec* h, dim3 ag, const AttnArgs& aa, int grp_rows_ub) {
  if (grp_rows_ub <= 8) launch_attn_r<KVT, 8>(h, ag, aa);
  else if (grp_rows_ub <= 16) launch_attn_r<KVT, 16>(h, ag, aa);
  else launch_attn_r<KVT, kAttnRows>(h, ag, aa);
}
void launch_attn(blt_dec* h, dim3 ag, const AttnArgs& aa, int grp_rows_ub) {
  if (h->kv_f32) launch_attn_t<float>(h, ag, aa, grp_rows_ub);
  else launch_attn_t<__nv_bfloat16>(h, ag, aa, grp_rows_ub);
}
template <typename KVT, int ROWS>
int set_attn_attrs_r(blt_dec* h) {
  const int smem = (int)attn_smem_bytes(h, ROWS);
  CK(cudaFuncSetAttribute(k_attn_partial<16, KVT, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  CK(cudaFuncSetAttribute(k_attn_partial<32, KVT, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  CK(cudaFuncSetAttribute(k_attn_partial<64, KVT, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  CK(cudaFuncSetAttribute(k_attn_partial<128, KVT, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  return BLT_OK;
}
template <typename KVT>
int set_attn_attrs(blt_dec* h) {
  TRY((set_attn_attrs_r<KVT, 8>(h)));
  TRY((set_attn_attrs_r<KVT, 16>(h)));
  TRY((set_attn_attrs_r<KVT, kAttnRows>(h)));
  return BLT_OK;
}

// ---------------------------------------------------------------------------- one decoder pass
// Runs every layer over the rows planned on the device (at most rows_ub rows,
// keys below keys_ub, at most groups_ub attention groups).
int run_pass_body(blt_dec* h, int rows_ub, int keys_ub, int groups_ub, bool want_head, int grp_rows_ub);
// grp_rows_ub: rows per attention group at most (a sequence's rows in the pass, capped at
// the planner's group size).
int run_pass(blt_dec* h, int rows_ub, int keys_ub, int groups_ub, bool want_head, int grp_rows_ub = kAttnRows) {
  return run_pass_body(h, rows_ub, keys_ub, groups_ub, want_head, std::min(grp_rows_ub, kAttnRows));
}
int run_pass_body(blt_dec* h, int rows_ub, int keys_ub, int groups_ub, bool want_head, int grp_rows_ub) {
  NvtxRange nvtx_("decoder pass (per-phase kernels)");
  const int d = h->d;
  // embed + per layer (cross add, attention partial + combine) + head statistics; GEMMs count themselves
  h->launches += 1 + 3 * (unsigned long long)h->L + (want_head ? 1 : 0);
  const int nb = std::max(1, std::min(rows_ub, 1024));
  k_embed<<<nb, 256, 0, h->stream>>>(h->rows, h->embed, h->h, d);
  AttnArgs aa = attn_args(h);
  const int nchunks = std::max(1, (keys_ub + h->CH - 1) / h->CH);
  for (int l = 0; l < h->L; ++l) {
    // B_l = D_{l-1} + W_o^c W_v^c o_lat
    k_cross_add<<<nb, 256, 0, h->stream>>>(h->rows, h->h, h->c_lat, h->cfg.max_latents, h->L, l, d);
    GemmArgs a = base_args(h);
    a.layer = l;
    a.X = h->h;
    a.ldx = d;
    a.gain = h->attn_norm[l];
    a.q = h->q;
    TRY(gemm<EPI_QKV>(h, h->qkv[l], a, rows_ub));
    aa.layer = l;
    launch_attn(h, dim3(h->H, nchunks, groups_ub), aa, grp_rows_ub);
    const dim3 cg(rows_ub, h->H);
    if (h->dh == 64) k_attn_combine<64><<<cg, 32, 0, h->stream>>>(aa);
    else if (h->dh == 32) k_attn_combine<32><<<cg, 32, 0, h->stream>>>(aa);
    else if (h->dh == 128) k_attn_combine<128><<<cg, 32, 0, h->stream>>>(aa);
    else k_attn_combine<16><<<cg, 32, 0, h->stream>>>(aa);
    CK(cudaGetLastError());
    a = base_args(h);
    a.layer = l;
    a.X = h->att;
    a.ldx = d;
    a.out = h->h;
    a.ldo = d;
    TRY(gemm<EPI_RESID>(h, h->o[l], a, rows_ub));
    a = base_args(h);
    a.layer = l;
    a.X = h->h;
    a.ldx = d;
    a.gain = h->ffn_norm[l];
    a.out = h->act;
    a.ldo = h->F;
    TRY(gemm<EPI_SWIGLU>(h, h->w13[l], a, rows_ub));
    a = base_args(h);
    a.layer = l;
    a.X = h->act;
    a.ldx = h->F;
    a.out = h->h;
    a.ldo = d;
    TRY(gemm<EPI_RESID>(h, h->w2[l], a, rows_ub));
  }
  if (want_head) {
    GemmArgs a = base_args(h);
    a.X = h->h;
    a.ldx = d;
    a.gain = h->final_norm;
    a.out = h->logits;
    a.ldo = 256;
    TRY(gemm<EPI_STORE>(h, h->head, a, rows_ub));
    k_head_stats<<<std::max(1, std::min((rows_ub + 7) / 8, 1024)), 256, 0, h->stream>>>(h->logits, h->rows.n_rows, h->conf,
                                                                                          h->pred, h->gap, h->ent);
  }
  CK(cudaGetLastError());
  return BLT_OK;
}

// ---------------------------------------------------------------------------- host bookkeeping
void refresh_bounds(blt_dec* h) {
  if (h->mirror_pending && cudaEventQuery(h->mirror_ev) == cudaSuccess) {
    const int B = h->cfg.max_batch;
    for (int s = 0; s < B; ++s) {
      h->kv_ub[s] = h->mirror[s];
      h->nlat_ub[s] = h->mirror[B + s];
    }
    h->mirror_pending = false;
  }
}

int post_mirror(blt_dec* h) {
  const int B = h->cfg.max_batch;
  CK(cudaMemcpyAsync(h->mirror, h->sd.kv_len, 2 * B * 4, cudaMemcpyDeviceToHost, h->stream));  // kv_len, n_lat
  CK(cudaEventRecord(h->mirror_ev, h->stream));
  h->mirror_pending = true;
  return BLT_OK;
}

// Make sure sequence s has KV pages for positions [0, need).
int ensure_pages(blt_dec* h, int s, int need, PageUpd& upd) {
  if (need > h->cfg.max_ctx) return fail(h, BLT_ERR_NO_SPACE, "sequence %d needs %d positions > max_ctx %d", s, need, h->cfg.max_ctx);
  while (h->seq_npages[s] * h->PT < need) {
    if (h->free_pages.empty()) return fail(h, BLT_ERR_NO_SPACE, "KV page pool exhausted");
    const int page = h->free_pages.back();
    h->free_pages.pop_back();
    const int idx = s * h->max_pages + h->seq_npages[s];
    h->pt_host[idx] = page;
    h->seq_npages[s]++;
    upd.idx[upd.n] = idx;
    upd.page[upd.n] = page;
    if (++upd.n == 64) {
      k_page_update<<<1, 64, 0, h->stream>>>(h->page_table, upd);
      h->launches += 1;
      upd.n = 0;
    }
  }
  return BLT_OK;
}

int flush_pages(blt_dec* h, PageUpd& upd) {
  if (upd.n) {
    k_page_update<<<1, 64, 0, h->stream>>>(h->page_table, upd);
    h->launches += 1;
  }
  upd.n = 0;
  CK(cudaGetLastError());
  return BLT_OK;
}

int make_desc(blt_dec* h, int batch, const int32_t* row_off, const int32_t* lat_off, CallDesc& cd) {
  if (batch < 1 || batch > h->cfg.max_batch || batch > kMaxCallBatch)
    return fail(h, BLT_ERR_INVALID_ARG, "batch %d outside 1..%d", batch, std::min(h->cfg.max_batch, kMaxCallBatch));
  cd.batch = batch;
  for (int s = 0; s <= batch; ++s) {
    cd.row_off[s] = row_off ? row_off[s] : 0;
    cd.lat_off[s] = lat_off ? lat_off[s] : 0;
    if (s > 0 && (cd.row_off[s] < cd.row_off[s - 1] || cd.lat_off[s] < cd.lat_off[s - 1]))
      return fail(h, BLT_ERR_INVALID_ARG, "offsets must be non-decreasing");
  }
  if (cd.row_off[0] != 0 || cd.lat_off[0] != 0) return fail(h, BLT_ERR_INVALID_ARG, "offsets must start at 0");
  return BLT_OK;
}

// Project new latents: c_l[slot] = W_o^c (W_v^c o) for every layer.
int project_latents(blt_dec* h, const CallDesc& cd, const float* new_lat, bool commit) {
  const int total = cd.lat_off[cd.batch];
  if (total == 0) return BLT_OK;
  if (!new_lat) return fail(h, BLT_ERR_INVALID_ARG, "new_latents is NULL but latent_offsets count %d", total);
  const int chunk = std::min(h->proj_rows, h->cfg.max_rows);
  const int LD = h->L * h->d;
  for (int r0 = 0; r0 < total; r0 += chunk) {
    const int r1 = std::min(total, r0 + chunk);
    k_lat_plan<<<1, 256, 0, h->stream>>>(cd, h->sd, h->lat_seq, h->lat_slot, h->n_lat_rows, r0, r1, commit ? 1 : 0,
                                         h->cfg.max_latents);
    h->launches += 1;
    // tmp[row][l*d + i] = (W_v^c of layer l) latent, every layer in one GEMM
    GemmArgs a = base_args(h);
    a.n_rows = nullptr;
    a.rows_host = r1 - r0;
    a.layer = 0;
    a.X = new_lat + (size_t)r0 * h->dg;
    a.ldx = h->dg;
    a.out = h->tmp;
    a.ldo = LD;
    TRY(gemm<EPI_STORE>(h, h->vc_all, a, r1 - r0));
    // c_lat[seq, slot, l] = (W_o^c of layer l) tmp[row][l*d ..]: tile group l reads column block l
    a.X = h->tmp;
    a.ldx = LD;
    a.group_tiles = h->d / 16;
    a.group_xoff = h->d;
    a.out = h->c_lat;
    a.lat_seq = h->lat_seq;
    a.lat_slot = h->lat_slot;
    TRY(gemm<EPI_LATC>(h, h->oc_all, a, r1 - r0));
  }
  CK(cudaGetLastError());
  return BLT_OK;
}

PlanArgs plan_args(blt_dec* h, int mode, int k) {
  PlanArgs p{};
  p.mode = mode;
  p.k = k;
  p.max_ctx = h->cfg.max_ctx;
  p.max_lat = h->cfg.max_latents;
  p.mask_id = h->V - 1;
  p.weight_bytes_per_pass = h->weight_bytes_per_pass;
  p.kv_bytes_per_key = h->kv_bytes_per_key;
  return p;
}

int plan(blt_dec* h, const PlanArgs& p, const CallDesc& cd) {
  h->launches += 1;
  k_plan<<<1, 256, 0, h->stream>>>(p, cd, h->sd, h->rows);
  CK(cudaGetLastError());
  return BLT_OK;
}

int groups_bound(const CallDesc& cd, int per_seq_extra) {
  int g = 0;
  for (int s = 0; s < cd.batch; ++s) g += (cd.row_off[s + 1] - cd.row_off[s] + per_seq_extra + 31) / 32;
  return std::max(g, 1);
}

int max_kv_ub(blt_dec* h, int batch) {
  int m = 0;
  for (int s = 0; s < batch; ++s) m = std::max(m, h->kv_ub[s]);
  return m;
}

// Bookkeeping kernels, greedy or (during a *_sampled call) drawing the committed bytes.
void launch_unmask(blt_dec* h, int batch, int k, float alpha, int step, float* out_logits) {
  if (h->samp_on)
    k_unmask_sampled<<<batch, 32, 0, h->stream>>>(h->sd, batch, k, alpha, step, h->sa, h->conf, h->pred, h->logits, out_logits,
                                                   h->eb ? h->ent : nullptr);
  else
    k_unmask<<<batch, 32, 0, h->stream>>>(h->sd, batch, k, alpha, step, h->conf, h->pred, h->logits, out_logits,
                                          h->eb ? h->ent : nullptr);
}
void launch_draft_ar(blt_dec* h, int batch, int step, float* out_logits) {
  if (h->samp_on)
    k_draft_ar_sampled<<<batch, 32, 0, h->stream>>>(h->sd, batch, step, h->sa, h->pred, h->logits, out_logits);
  else
    k_draft_ar<<<batch, 32, 0, h->stream>>>(h->sd, batch, step, h->pred, h->logits, out_logits);
}

// Fill k-byte blocks (BLT-D / BLT-DV draft) with the pending rows in pass 1.
int block_loop(blt_dec* h, const CallDesc& cd, const blt_rows_in* pend, int k, float alpha, int max_steps, float* out_logits) {
  const int batch = cd.batch;
  const int np_total = cd.row_off[batch];
  const int rows1 = np_total + batch * k;
  int npmax = 0;
  for (int s = 0; s < batch; ++s) npmax = std::max(npmax, cd.row_off[s + 1] - cd.row_off[s]);
  const int keys_ub = max_kv_ub(h, batch) + npmax + k;
  PlanArgs p = plan_args(h, PL_FIRST, k);
  p.pend_bytes = pend->bytes;
  p.pend_lat = pend->row_latent;
  TRY(plan(h, p, cd));
  TRY(run_pass(h, rows1, keys_ub, groups_bound(cd, k), true, npmax + k));
  launch_unmask(h, batch, k, alpha, 0, out_logits);
  h->launches += 1;
  for (int st = 1; st < max_steps; ++st) {
    PlanArgs pb = plan_args(h, PL_BLOCK, k);
    TRY(plan(h, pb, cd));
    TRY(run_pass(h, batch * k, keys_ub, batch * ((k + 31) / 32), true, k));
    launch_unmask(h, batch, k, alpha, st, out_logits);
    h->launches += 1;
  }
  CK(cudaGetLastError());
  return BLT_OK;
}

int mega_run(blt_dec* h, int mode, int batch, int k, float alpha, int max_passes, int rows_ub, const int* vlat, float* out_logits,
             int* out_acc, unsigned char* out_next);
bool use_mega(const blt_dec* h, int rows_ub, int batch);

// The block loop on the persistent kernel when the pass is small enough.
int diffuse_passes(blt_dec* h, const CallDesc& cd, const blt_rows_in* pend, int k, float alpha, int max_steps, float* out_logits) {
  const int batch = cd.batch;
  // a position's confidence (its largest byte probability) is at least 1/V: with alpha <= 1/V
  // every masked position commits in the first pass, and the later passes would have no rows
  if (!h->eb && alpha * (float)h->V <= 1.f) max_steps = 1;
  const int rows1 = cd.row_off[batch] + batch * k;
  if (!use_mega(h, rows1, batch)) return block_loop(h, cd, pend, k, alpha, max_steps, out_logits);
  PlanArgs p = plan_args(h, PL_FIRST, k);
  p.pend_bytes = pend->bytes;
  p.pend_lat = pend->row_latent;
  TRY(plan(h, p, cd));
  return mega_run(h, MM_DIFFUSE, batch, k, alpha, max_steps, rows1, nullptr, out_logits, nullptr, nullptr);
}

int check_pending(blt_dec* h, const blt_rows_in* r, bool need_rows) {
  if (!r) return fail(h, BLT_ERR_INVALID_ARG, "rows is NULL");
  if (need_rows && !r->row_offsets) return fail(h, BLT_ERR_INVALID_ARG, "row_offsets is NULL");
  return BLT_OK;
}

int reserve(blt_dec* h, const CallDesc& cd, int extra_positions, bool lat_commit) {
  PageUpd upd{};
  for (int s = 0; s < cd.batch; ++s) {
    const int np = cd.row_off[s + 1] - cd.row_off[s];
    const int nl = cd.lat_off[s + 1] - cd.lat_off[s];
    TRY(ensure_pages(h, s, h->kv_ub[s] + np + extra_positions, upd));
    if (h->nlat_ub[s] + nl > h->cfg.max_latents)
      return fail(h, BLT_ERR_NO_SPACE, "sequence %d latent slots %d + %d > max_latents %d", s, h->nlat_ub[s], nl,
                  h->cfg.max_latents);
  }
  (void)lat_commit;
  return flush_pages(h, upd);
}

void bump_bounds(blt_dec* h, const CallDesc& cd, int extra_kv) {
  for (int s = 0; s < cd.batch; ++s) {
    h->kv_ub[s] += cd.row_off[s + 1] - cd.row_off[s] + extra_kv;
    h->nlat_ub[s] += cd.lat_off[s + 1] - cd.lat_off[s];
  }
}

__global__ void k_snapshot_base(SeqDev sd, int batch) {
  const int s = threadIdx.x + blockIdx.x * blockDim.x;
  if (s < batch) sd.kv_base[s] = sd.kv_len[s];
}
__global__ void k_finish_prefill(SeqDev sd, CallDesc cd) {
  const int s = threadIdx.x;
  if (s < cd.batch) sd.kv_len[s] = sd.kv_base[s] + (cd.row_off[s + 1] - cd.row_off[s]);
}
__global__ void k_copy_logits(const float* src, float* dst, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) dst[i] = src[i];
}

// ---------------------------------------------------------------------------- persistent pass kernel
template <int NG, int PL, int DH, typename KVT>
size_t mega_smem(const blt_dec* h) {
  (void)h;
  const size_t red = (size_t)kMaxPieces * 8 * 16 * 8 * NG * 4;
  const size_t att = (size_t)(kMegaRows * DH + kMegaRows * 128) * 4;
  return (size_t)kRingSlots * kSlotBytes + std::max(red, att) + 8 * 8 * kMegaMaxNG * 4 + 2 * (size_t)kMaxPieces * kMegaRows * 16 * 4 +
         1024 * 4;  // ring, reduction / attention scratch, ssr, hpre, cpre, gain (d <= 1024)
}

template <int NG, int PL, int DH, typename KVT>
int mega_prepare_t(blt_dec* h) {
  const size_t smem = mega_smem<NG, PL, DH, KVT>(h);
  CK(cudaFuncSetAttribute(k_mega<NG, PL, DH, KVT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int per_sm = 0;
  CK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_mega<NG, PL, DH, KVT>, kMegaThreads, smem));
  if (per_sm < 1) return fail(h, BLT_ERR_CUDA, "persistent pass kernel does not fit on an SM");
  return BLT_OK;
}

template <int PL, int DH, typename KVT>
int mega_prepare_pd(blt_dec* h) {
  TRY((mega_prepare_t<1, PL, DH, KVT>(h)));
  return mega_prepare_t<2, PL, DH, KVT>(h);
}

// Decide whether the persistent kernel applies to this model and set it up.
int mega_setup(blt_dec* h) {
  const int es = h->kv_f32 ? 4 : 2;
  const int nseg = h->F > kSegCols ? h->F / kSegCols : 1;
  if (!(h->cfg.flags & BLT_FLAG_PERSISTENT) || h->d > 1024 || h->d % 128 != 0 || h->F % 128 != 0 || h->F > 4096 ||
      (h->F > kSegCols && h->F % kSegCols != 0) || (h->dh != 32 && h->dh != 64) || h->CH != 128 || 128 % h->PT != 0 ||
      2 * h->CH * h->dh * es > kSlotBytes)
    return BLT_OK;
  int dev = 0;
  CK(cudaGetDevice(&dev));
  int coop = 0;
  CK(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev));
  CK(cudaDeviceGetAttribute(&h->nsm, cudaDevAttrMultiProcessorCount, dev));
  if (!coop || h->nsm < nseg) return BLT_OK;
  int rc;
  if (h->planes == 1) {
    rc = h->kv_f32 ? (h->dh == 64 ? mega_prepare_pd<1, 64, float>(h) : mega_prepare_pd<1, 32, float>(h))
                   : (h->dh == 64 ? mega_prepare_pd<1, 64, __nv_bfloat16>(h) : mega_prepare_pd<1, 32, __nv_bfloat16>(h));
  } else {
    rc = h->kv_f32 ? (h->dh == 64 ? mega_prepare_pd<2, 64, float>(h) : mega_prepare_pd<2, 32, float>(h))
                   : (h->dh == 64 ? mega_prepare_pd<2, 64, __nv_bfloat16>(h) : mega_prepare_pd<2, 32, __nv_bfloat16>(h));
  }
  if (rc != BLT_OK) {
    fprintf(stderr, "bltdec: persistent pass kernel unavailable (%s); using per-phase kernels\n", h->err.c_str());
    h->err.clear();
    return BLT_OK;
  }
  std::vector<LayerW> lw(h->L);
  for (int l = 0; l < h->L; ++l)
    lw[l] = LayerW{h->qkv[l].w, h->o[l].w, h->w13[l].w, h->w2[l].w, h->attn_norm[l], h->ffn_norm[l]};
  TRY(dalloc(h, &h->d_layers, h->L));
  CK(cudaMemcpy(h->d_layers, lw.data(), sizeof(LayerW) * h->L, cudaMemcpyHostToDevice));
  // exchange words: [rows][d] x5 (stream, q, k, v, attention), [rows][F], [nseg-1][rows][d], [rows][256],
  // and the chunk partials [rows][H][CMAX][2 + dh]
  const size_t R = kMegaRows, d = h->d;
  h->x_cmax = (h->cfg.max_ctx + h->CH - 1) / h->CH;
  const size_t n_part = R * h->H * (size_t)h->x_cmax * (2 + h->dh);
  h->xbuf_words = 5 * R * d + R * h->F + (size_t)std::max(nseg - 1, 1) * R * d + R * 256 + n_part;
  TRY(dalloc(h, &h->xbuf, h->xbuf_words));
  CK(cudaMemset(h->xbuf, 0, h->xbuf_words * 8));
  unsigned long long* p = h->xbuf;
  h->x_h = p, p += R * d;
  h->x_q = p, p += R * d;
  h->x_k = p, p += R * d;
  h->x_v = p, p += R * d;
  h->x_att = p, p += R * d;
  h->x_act = p, p += R * h->F;
  h->x_w2p = p, p += (size_t)std::max(nseg - 1, 1) * R * d;
  h->x_logit = p, p += R * 256;
  h->x_part = p;
  TRY(dalloc(h, &h->flags, 3));  // [0] pass plan word, [1] pass-end arrivals, [2] abort word
  CK(cudaMemset(h->flags, 0, 12));
  TRY(dalloc(h, &h->dec_val, 1));
  h->abort_flag = reinterpret_cast<int*>(h->flags + 2);
  h->epoch = 1;
  h->mega_ok = true;
  if (const char* ip = getenv("BLTDEC_MEGA_ITEMS_PER_SM")) h->mega_items_per_sm = std::max(0, atoi(ip));
  if (const char* sp = getenv("BLTDEC_SPIN_NS")) {
    unsigned a = 0, b = 0;
    if (sscanf(sp, "%u,%u", &a, &b) == 2 && a <= 100000 && b <= 100000) h->spin_ns[0] = a, h->spin_ns[1] = b;
  }
  if (const char* tp = getenv("BLTDEC_TRACE")) {
    h->trace_path = tp;
    TRY(dalloc(h, &h->trace, (size_t)h->nsm * kTraceEvents));
    CK(cudaMemset(h->trace, 0, (size_t)h->nsm * kTraceEvents * 8));
  }
  return BLT_OK;
}

// The persistent kernel runs a CTA's attention items one after another, each with a fixed
// latency of a few microseconds; with many long sequences (batch 16 at 4096 cached bytes:
// ~57 items per CTA per layer) the per-phase kernels, whose attention blocks overlap on
// every SM, are faster (measured 18 vs 25 ms per 8-pass draft call there, while at batch 1
// and 1024 bytes the persistent kernel is 2.5x faster).  Above 8 items per SM (the knob
// below): per-phase.
bool use_mega(const blt_dec* h, int rows_ub, int batch) {
  if (!h->mega_ok || h->samp_on || rows_ub > kMegaRows || batch > kMegaRows) return false;
  long long items = 0;
  const int per_seq = (rows_ub + batch - 1) / batch;
  for (int s = 0; s < batch; ++s) items += (long long)h->H * ((h->kv_ub[s] + per_seq + h->CH - 1) / h->CH);
  return items <= (long long)h->mega_items_per_sm * h->nsm;
}

template <int NG, int PL, int DH, typename KVT>
int mega_launch_t(blt_dec* h, MegaArgs& m) {
  const size_t smem = mega_smem<NG, PL, DH, KVT>(h);
  void* args[] = {&m};
  CK(cudaLaunchCooperativeKernel((const void*)k_mega<NG, PL, DH, KVT>, dim3(h->nsm), dim3(kMegaThreads), args, smem, h->stream));
  h->launches += 1;
  h->persistent_calls += 1;
  return BLT_OK;
}

// All passes of one call in one launch (rows of pass 1 already planned).
int mega_run(blt_dec* h, int mode, int batch, int k, float alpha, int max_passes, int rows_ub, const int* vlat, float* out_logits,
             int* out_acc, unsigned char* out_next) {
  NvtxRange nvtx_("decoder passes (persistent kernel, one launch)");
  MegaArgs m{};
  m.layers = h->d_layers;
  m.whead = h->head.w;
  m.final_norm = h->final_norm;
  m.L = h->L;
  m.d = h->d;
  m.H = h->H;
  m.dh = h->dh;
  m.F = h->F;
  m.planes = h->planes;
  m.eps = h->cfg.norm_eps;
  m.ga = base_args(h);
  m.aa = attn_args(h);
  m.rows = h->rows;
  m.sd = h->sd;
  m.x_h = h->x_h;
  m.x_q = h->x_q;
  m.x_k = h->x_k;
  m.x_v = h->x_v;
  m.x_part = h->x_part;
  m.x_att = h->x_att;
  m.x_act = h->x_act;
  m.x_w2p = h->x_w2p;
  m.x_logit = h->x_logit;
  m.CMAX = h->x_cmax;
  m.logits = h->logits;
  m.conf = h->conf;
  m.ent = h->ent;
  m.eb = h->eb;
  m.pred = h->pred;
  m.gap = h->gap;
  m.flags = h->flags;
  m.dec_val = h->dec_val;
  // epochs: unique per (call, pass, layer, stage); restart from zeroed words long before they wrap
  const unsigned span = (unsigned)(max_passes + 1) * (unsigned)(h->L + 1) * 8u + 16u;
  if (h->epoch > 0xF0000000u - span) {
    CK(cudaMemsetAsync(h->xbuf, 0, h->xbuf_words * 8, h->stream));
    CK(cudaMemsetAsync(h->flags, 0, 8, h->stream));
    h->epoch = 1;
  }
  m.epoch0 = h->epoch;
  h->epoch += span;
  CK(cudaMemsetAsync(h->flags + 1, 0, 8, h->stream));  // pass-end arrivals and abort word of this launch
  m.abort = h->abort_flag;
  const bool stall = (h->cfg.flags & BLT_FLAG_TEST_STALL) != 0;
  m.wait_ns = stall ? 2000000ull : 500000000ull;  // 2 ms under the test-only stall, else 0.5 s
  m.spin_ns0 = h->spin_ns[0];
  m.spin_ns1 = h->spin_ns[1];
  m.stall_test = stall ? 1 : 0;
  m.trace = h->trace;
  if (h->trace) {
    h->trace_pending = 1;
  }
  m.mode = mode;
  m.batch = batch;
  m.k = k;
  m.max_passes = max_passes;
  m.alpha = alpha;
  m.vlat = vlat;
  m.out_logits = out_logits;
  m.out_acc = out_acc;
  m.out_next = out_next;
  m.plan = plan_args(h, PL_BLOCK, k);
  const bool ng1 = rows_ub <= 8;
  if (h->planes == 1) {
    if (h->kv_f32) {
      if (h->dh == 64) return ng1 ? mega_launch_t<1, 1, 64, float>(h, m) : mega_launch_t<2, 1, 64, float>(h, m);
      return ng1 ? mega_launch_t<1, 1, 32, float>(h, m) : mega_launch_t<2, 1, 32, float>(h, m);
    }
    if (h->dh == 64) return ng1 ? mega_launch_t<1, 1, 64, __nv_bfloat16>(h, m) : mega_launch_t<2, 1, 64, __nv_bfloat16>(h, m);
    return ng1 ? mega_launch_t<1, 1, 32, __nv_bfloat16>(h, m) : mega_launch_t<2, 1, 32, __nv_bfloat16>(h, m);
  }
  if (h->kv_f32) {
    if (h->dh == 64) return ng1 ? mega_launch_t<1, 2, 64, float>(h, m) : mega_launch_t<2, 2, 64, float>(h, m);
    return ng1 ? mega_launch_t<1, 2, 32, float>(h, m) : mega_launch_t<2, 2, 32, float>(h, m);
  }
  if (h->dh == 64) return ng1 ? mega_launch_t<1, 2, 64, __nv_bfloat16>(h, m) : mega_launch_t<2, 2, 64, __nv_bfloat16>(h, m);
  return ng1 ? mega_launch_t<1, 2, 32, __nv_bfloat16>(h, m) : mega_launch_t<2, 2, 32, __nv_bfloat16>(h, m);
}

// Body of blt_dec_prefill after argument checks (cd made, bounds refreshed).
int prefill_impl(blt_dec* h, int batch, const blt_rows_in* rows, float* out_logits, const CallDesc& cd) {
  const int total = cd.row_off[batch];
  TRY(reserve(h, cd, 0, true));
  h->calls += 1;
  TRY(project_latents(h, cd, rows->new_latents, true));
  k_snapshot_base<<<1, 256, 0, h->stream>>>(h->sd, batch);
  h->launches += 1;
  int kmax = 0;
  for (int s = 0; s < batch; ++s) kmax = std::max(kmax, h->kv_ub[s] + cd.row_off[s + 1] - cd.row_off[s]);
  const int chunk = h->cfg.max_rows;
  for (int r0 = 0; r0 < total; r0 += chunk) {
    const int r1 = std::min(total, r0 + chunk);
    PlanArgs p = plan_args(h, PL_PREFILL, 0);
    p.r0 = r0;
    p.r1 = r1;
    p.pend_bytes = rows->bytes;
    p.pend_lat = rows->row_latent;
    TRY(plan(h, p, cd));
    TRY(run_pass(h, r1 - r0, kmax, (r1 - r0 + 31) / 32 + batch, out_logits != nullptr));
    if (out_logits) {
      k_copy_logits<<<256, 256, 0, h->stream>>>(h->logits, out_logits + (size_t)r0 * 256, (r1 - r0) * 256);
      h->launches += 1;
    }
  }
  k_finish_prefill<<<1, 256, 0, h->stream>>>(h->sd, cd);
  h->launches += 1;
  CK(cudaGetLastError());
  bump_bounds(h, cd, 0);
  return post_mirror(h);
}

}  // namespace


// ============================================================================ prefill without allocation
// One file-scope device arena holds the per-call scratch of blt_dec_prefill_noalloc:
// activations, attention partials, logits, the row plan and the latent temporary
// for chunks of at most kNaRows rows over at most kNaKeys key positions.
namespace {
constexpr int kNaRows = 32;
constexpr int kNaKeys = 4096;
constexpr int kNaMaxD = 1024, kNaMaxF = 4096, kNaMaxH = 16, kNaMaxDh = 64, kNaChunk = 128;
constexpr int kNaCMax = kNaKeys / kNaChunk;
constexpr int kNaGroups = kNaRows / kAttnRows + kMaxCallBatch + 1;
constexpr size_t na_align(size_t x) { return (x + 255) & ~(size_t)255; }
constexpr size_t kNaArenaBytes =
    na_align(4ull * kNaRows * kNaMaxD * 4) * 1 + na_align((size_t)kNaRows * kNaMaxF * 4) + na_align((size_t)kNaRows * 256 * 4) +
    na_align((size_t)kNaRows * kNaMaxH * kNaCMax * 8) + na_align((size_t)kNaRows * kNaMaxH * kNaCMax * kNaMaxDh * 4) +
    4 * na_align(kNaRows * 4) + 5 * na_align(kNaRows * 4 + 4) + 5 * na_align(kNaGroups * 4 + 4) + 3 * na_align(kNaRows * 4 + 4) + 16 * 256;
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_arena[kNaArenaBytes];

namespace {
std::mutex g_na_mutex;
void* g_na_base[256];  // device address of the arena, per device (resolved on first use)

// Address of the arena on the current device; resolved once per device.
int na_arena(blt_dec* h, unsigned char** out) {
  int dev = 0;
  CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 256) return fail(h, BLT_ERR_CUDA, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_na_mutex);
  if (!g_na_base[dev]) {
    void* p = nullptr;
    CK(cudaGetSymbolAddress(&p, g_noalloc_arena));
    g_na_base[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_na_base[dev]);
  return BLT_OK;
}

struct NaCarve {
  unsigned char* base;
  size_t off = 0;
  template <class T>
  T* take(size_t n) {
    off = na_align(off);
    T* p = reinterpret_cast<T*>(base + off);
    off += n * sizeof(T);
    return p;
  }
};

// Points the handle's pass scratch at the arena for one call and restores it after.
struct NaSwap {
  blt_dec* h;
  float *hh, *q, *att, *act, *logits, *tmp, *conf, *gap, *ent;
  float2* part_ml;
  float* part_o;
  int* pred;
  RowsDev rows;
  int *lat_seq, *lat_slot, *n_lat_rows;
  int cmax, max_rows, proj_rows;
  NaSwap(blt_dec* hd, unsigned char* base) : h(hd) {
    hh = h->h, q = h->q, att = h->att, act = h->act, logits = h->logits, tmp = h->tmp, conf = h->conf, gap = h->gap, ent = h->ent;
    part_ml = h->part_ml, part_o = h->part_o, pred = h->pred, rows = h->rows;
    lat_seq = h->lat_seq, lat_slot = h->lat_slot, n_lat_rows = h->n_lat_rows, cmax = h->CMAX, max_rows = h->cfg.max_rows;
    proj_rows = h->proj_rows;
    NaCarve c{base};
    h->h = c.take<float>((size_t)kNaRows * kNaMaxD);
    h->q = c.take<float>((size_t)kNaRows * kNaMaxD);
    h->att = c.take<float>((size_t)kNaRows * kNaMaxD);
    h->tmp = c.take<float>((size_t)kNaRows * kNaMaxD);
    h->act = c.take<float>((size_t)kNaRows * kNaMaxF);
    h->logits = c.take<float>((size_t)kNaRows * 256);
    h->part_ml = c.take<float2>((size_t)kNaRows * kNaMaxH * kNaCMax);
    h->part_o = c.take<float>((size_t)kNaRows * kNaMaxH * kNaCMax * kNaMaxDh);
    h->conf = c.take<float>(kNaRows);
    h->gap = c.take<float>(kNaRows);
    h->ent = c.take<float>(kNaRows);
    h->pred = c.take<int>(kNaRows);
    RowsDev& r = h->rows;
    r.seq = c.take<int>(kNaRows);
    r.pos = c.take<int>(kNaRows);
    r.lat = c.take<int>(kNaRows);
    r.nkeys = c.take<int>(kNaRows);
    r.byte = c.take<int>(kNaRows);
    r.n_rows = c.take<int>(1);
    r.g_seq = c.take<int>(kNaGroups);
    r.g_row0 = c.take<int>(kNaGroups);
    r.g_nrows = c.take<int>(kNaGroups);
    r.g_kmax = c.take<int>(kNaGroups);
    r.g_fresh = c.take<int>(kNaGroups);
    r.n_groups = c.take<int>(1);
    h->lat_seq = c.take<int>(kNaRows);
    h->lat_slot = c.take<int>(kNaRows);
    h->n_lat_rows = c.take<int>(1);
    h->CMAX = kNaCMax;
    h->cfg.max_rows = kNaRows;
    h->proj_rows = (int)((size_t)kNaRows * kNaMaxD / ((size_t)h->L * h->d));  // tmp holds rows x L*d; >= 1 (L*d checked)
    used = c.off;
  }
  size_t used = 0;
  ~NaSwap() {
    h->h = hh, h->q = q, h->att = att, h->act = act, h->logits = logits, h->tmp = tmp, h->conf = conf, h->gap = gap, h->ent = ent;
    h->part_ml = part_ml, h->part_o = part_o, h->pred = pred, h->rows = rows;
    h->lat_seq = lat_seq, h->lat_slot = lat_slot, h->n_lat_rows = n_lat_rows, h->CMAX = cmax, h->cfg.max_rows = max_rows;
    h->proj_rows = proj_rows;
  }
};
}  // namespace

// ============================================================================ C ABI
extern "C" {

int blt_dec_init(const blt_dec_config* cfg, const blt_dec_weights* w, void* cuda_stream, blt_dec_t** out) {
  NvtxRange nvtx_("blt_dec_init");
  if (!cfg || !w || !out) return BLT_ERR_INVALID_ARG;
  *out = nullptr;
  blt_dec* h = new blt_dec();
  h->cfg = *cfg;
  auto bad = [&](const char* msg) {
    blt_dec_free(h);
    return BLT_ERR_INVALID_ARG;
  };
  const blt_dec_config& c = *cfg;
  if (c.n_layers < 1 || c.d_model < 128 || c.d_model % 128 || c.n_heads < 1 || c.d_model % c.n_heads ||
      (c.d_model / c.n_heads) % 16 || c.d_model / c.n_heads > 128 || c.d_ffn % 128 || c.d_ffn < 128 || c.d_global % 128 ||
      c.d_global < 128 || c.vocab != 257 || (c.weight_dtype != BLT_W_F32 && c.weight_dtype != BLT_W_BF16) ||
      c.max_batch < 1 || c.max_batch > kMaxCallBatch || c.max_ctx < 2 || c.max_latents < 1 || c.max_rows < 1 ||
      c.max_block < 1 || c.max_block > kMaxBlock || c.page_tokens < 16 || c.page_tokens % 16 || !(c.norm_eps > 0) ||
      !(c.rope_theta > 0) || !w->embed || !w->head || !w->final_norm || !w->layer)
    return bad("config");
  const int dhh = c.d_model / c.n_heads;
  if (dhh != 16 && dhh != 32 && dhh != 64 && dhh != 128) return bad("head dim");
  h->L = c.n_layers;
  h->d = c.d_model;
  h->H = c.n_heads;
  h->dh = dhh;
  h->F = c.d_ffn;
  h->dg = c.d_global;
  h->V = c.vocab;
  h->planes = c.weight_dtype == BLT_W_F32 ? 2 : 1;
  h->PT = c.page_tokens;
  h->max_pages = (c.max_ctx + h->PT - 1) / h->PT;
  h->n_pages = c.kv_pages > 0 ? c.kv_pages : c.max_batch * h->max_pages;
  h->CH = c.attn_chunk > 0 ? c.attn_chunk : 128;
  if (h->CH > 128 || h->CH % 16) return bad("attn_chunk");
  h->CMAX = (c.max_ctx + h->CH - 1) / h->CH;

  int rc = BLT_OK;
  auto run = [&]() -> int {
    if (cuda_stream) {
      h->stream = (cudaStream_t)cuda_stream;
    } else {
      CK(cudaStreamCreateWithFlags(&h->stream, cudaStreamNonBlocking));
      h->own_stream = true;
    }
    const int d = h->d, dg = h->dg, F = h->F, L = h->L, dh = h->dh, pl = h->planes;
    h->tc = (c.flags & BLT_FLAG_TENSOR_CORES) && pl == 1 && c.max_rows >= kTcMinRows && d % kTcBK == 0 && F % kTcBK == 0;
    h->qkv.resize(L);
    h->o.resize(L);
    h->w13.resize(L);
    h->w2.resize(L);
    h->attn_norm.resize(L);
    h->ffn_norm.resize(L);
    for (int l = 0; l < L; ++l) {
      const float* const* lw = w->layer + (size_t)l * BLT_LAYER_NT;
      for (int t = 0; t < BLT_LAYER_NT; ++t)
        if (!lw[t] && t != BLT_LAYER_WQ_C && t != BLT_LAYER_WK_C && t != BLT_LAYER_NORM_C)
          return fail(h, BLT_ERR_INVALID_ARG, "layer %d tensor %d is NULL", l, t);
      const float* wqkv = lw[BLT_LAYER_WQKV];
      // q and k rows are grouped so that each 16-row tile holds 8 rotary pairs (j, j + dh/2)
      TRY(pack_matrix(h, h->qkv[l], 3 * d, d, pl, [&](int r) -> const float* {
        const int sec = r / d, rr = r % d;
        if (sec == 2) return wqkv + (size_t)r * d;
        const int tph = dh / 16;
        const int tile = rr / 16, r16 = rr % 16;
        const int head = tile / tph, tt = tile % tph;
        const int j = tt * 8 + (r16 & 7) + (r16 >= 8 ? dh / 2 : 0);
        return wqkv + ((size_t)sec * d + head * dh + j) * d;
      }, true));
      TRY(pack_matrix(h, h->o[l], d, d, pl, [&](int r) { return lw[BLT_LAYER_WO] + (size_t)r * d; }, true));
      // SwiGLU: tile rows 0..7 = W1 rows j..j+7, rows 8..15 = the same rows of W3
      TRY(pack_matrix(h, h->w13[l], 2 * F, d, pl, [&](int r) -> const float* {
        const int tile = r / 16, r16 = r % 16;
        const int j = tile * 8 + (r16 & 7);
        return (r16 < 8 ? lw[BLT_LAYER_W1] : lw[BLT_LAYER_W3]) + (size_t)j * d;
      }, true));
      TRY(pack_matrix(h, h->w2[l], d, F, pl, [&](int r) { return lw[BLT_LAYER_W2] + (size_t)r * F; }, true));
      TRY(upload(h, &h->attn_norm[l], lw[BLT_LAYER_ATTN_NORM], d));
      TRY(upload(h, &h->ffn_norm[l], lw[BLT_LAYER_FFN_NORM], d));
    }
    // one projection GEMM per matrix kind covers every layer
    TRY(pack_matrix(h, h->vc_all, L * d, dg, pl,
                    [&](int r) { return w->layer[(size_t)(r / d) * BLT_LAYER_NT + BLT_LAYER_WV_C] + (size_t)(r % d) * dg; }));
    TRY(pack_matrix(h, h->oc_all, L * d, d, pl,
                    [&](int r) { return w->layer[(size_t)(r / d) * BLT_LAYER_NT + BLT_LAYER_WO_C] + (size_t)(r % d) * d; }));
    TRY(pack_matrix(h, h->head, 256, d, pl, [&](int r) { return w->head + (size_t)r * d; }, true));
    {
      // the embedding is read once per row: keep it fp32, values rounded like the weights
      std::vector<float> e((size_t)h->V * d);
      for (size_t i = 0; i < e.size(); ++i) {
        const float v = w->embed[i];
        e[i] = (pl == 1) ? bf16_to_f(bf16_rne(v)) : v;
      }
      TRY(upload(h, &h->embed, e.data(), e.size()));
    }
    TRY(upload(h, &h->final_norm, w->final_norm, d));
    {
      const int half = dh / 2;
      std::vector<float> cs((size_t)c.max_ctx * half), sn((size_t)c.max_ctx * half);
      for (int p = 0; p < c.max_ctx; ++p)
        for (int i = 0; i < half; ++i) {
          const double ang = (double)p * std::pow((double)c.rope_theta, -2.0 * i / dh);
          cs[(size_t)p * half + i] = (float)std::cos(ang);
          sn[(size_t)p * half + i] = (float)std::sin(ang);
        }
      TRY(upload(h, &h->rope_cos, cs.data(), cs.size()));
      TRY(upload(h, &h->rope_sin, sn.data(), sn.size()));
    }
    h->weight_bytes_per_pass = h->head.bytes();
    for (int l = 0; l < L; ++l)
      h->weight_bytes_per_pass += h->qkv[l].bytes() + h->o[l].bytes() + h->w13[l].bytes() + h->w2[l].bytes();
    h->kv_bytes_per_key = (unsigned long long)L * 2 * d * (pl == 2 ? 4 : 2);
    // KV pool [pages][L][2][H][PT][dh]: bf16 for bf16 weights, fp32 for fp32 weights
    h->kv_f32 = pl == 2;
    {
      char* kvp = nullptr;
      TRY(dalloc(h, &kvp, (size_t)h->n_pages * L * 2 * d * h->PT * (h->kv_f32 ? 4 : 2)));
      h->kv = kvp;
    }
    TRY(dalloc(h, &h->page_table, (size_t)c.max_batch * h->max_pages));
    CK(cudaMemset(h->page_table, 0xFF, (size_t)c.max_batch * h->max_pages * 4));
    h->pt_host.assign((size_t)c.max_batch * h->max_pages, -1);
    h->free_pages.resize(h->n_pages);
    for (int i = 0; i < h->n_pages; ++i) h->free_pages[i] = h->n_pages - 1 - i;
    h->seq_npages.assign(c.max_batch, 0);
    TRY(dalloc(h, &h->c_lat, (size_t)c.max_batch * c.max_latents * L * d));
    const int R = c.max_rows;
    const int RL = std::max(R, c.max_batch * c.max_block + R);
    TRY(dalloc(h, &h->h, (size_t)RL * d));
    TRY(dalloc(h, &h->rs, RL));
    TRY(dalloc(h, &h->q, (size_t)RL * d));
    TRY(dalloc(h, &h->att, (size_t)RL * d));
    TRY(dalloc(h, &h->act, (size_t)RL * F));
    TRY(dalloc(h, &h->logits, (size_t)RL * 256));
    TRY(dalloc(h, &h->tmp, (size_t)R * L * d));
    h->proj_rows = R;
    TRY(dalloc(h, &h->part_ml, (size_t)RL * h->H * h->CMAX));
    TRY(dalloc(h, &h->part_o, (size_t)RL * h->H * h->CMAX * dh));
    TRY(dalloc(h, &h->conf, RL));
    TRY(dalloc(h, &h->gap, RL));
    TRY(dalloc(h, &h->ent, RL));
    TRY(dalloc(h, &h->pred, RL));
    RowsDev& rd = h->rows;
    TRY(dalloc(h, &rd.seq, RL));
    TRY(dalloc(h, &rd.pos, RL));
    TRY(dalloc(h, &rd.lat, RL));
    TRY(dalloc(h, &rd.nkeys, RL));
    TRY(dalloc(h, &rd.byte, RL));
    TRY(dalloc(h, &rd.n_rows, 1));
    TRY(dalloc(h, &rd.g_seq, RL + c.max_batch));
    TRY(dalloc(h, &rd.g_row0, RL + c.max_batch));
    TRY(dalloc(h, &rd.g_nrows, RL + c.max_batch));
    TRY(dalloc(h, &rd.g_kmax, RL + c.max_batch));
    TRY(dalloc(h, &rd.g_fresh, RL + c.max_batch));
    TRY(dalloc(h, &rd.n_groups, 1));
    TRY(dalloc(h, &h->lat_seq, R));
    TRY(dalloc(h, &h->lat_slot, R));
    TRY(dalloc(h, &h->n_lat_rows, 1));
    SeqDev& sd = h->sd;
    const int B = c.max_batch;
    TRY(dalloc(h, &sd.kv_len, 2 * B));  // kv_len then n_lat: the host mirror reads both in one copy
    sd.n_lat = sd.kv_len + B;
    TRY(dalloc(h, &sd.kv_base, B));
    TRY(dalloc(h, &sd.active, B));
    TRY(dalloc(h, &sd.steps, B));
    TRY(dalloc(h, &sd.y_last, B));
    TRY(dalloc(h, &sd.last_row, B));
    TRY(dalloc(h, &sd.blk_row, (size_t)B * kMaxBlock));
    TRY(dalloc(h, &sd.blk, (size_t)B * kMaxBlock));
    TRY(dalloc(h, &sd.masked, (size_t)B * kMaxBlock));
    TRY(dalloc(h, &sd.status, 1));
    TRY(dalloc(h, &sd.counters, 8));
    TRY(dalloc(h, &h->sa.qdist, (size_t)B * kMaxBlock * 256));
    TRY(dalloc(h, &h->sa.p0dist, (size_t)B * 256));
    TRY(dalloc(h, &h->sa.pdist, (size_t)B * 256));
    CK(cudaMemset(sd.kv_len, 0, B * 4));
    CK(cudaMemset(sd.n_lat, 0, B * 4));
    CK(cudaMemset(sd.active, 0, B * 4));
    CK(cudaMemset(sd.status, 0, 4));
    CK(cudaMemset(sd.counters, 0, 64));
    CK(cudaMemset(sd.blk, 0, (size_t)B * kMaxBlock));
    CK(cudaMemset(sd.masked, 0, (size_t)B * kMaxBlock));
    CK(cudaMemset(h->c_lat, 0, (size_t)c.max_batch * c.max_latents * L * d * 4));
    CK(cudaHostAlloc((void**)&h->mirror, 2 * B * 4, cudaHostAllocDefault));
    CK(cudaEventCreateWithFlags(&h->mirror_ev, cudaEventDisableTiming));
    h->kv_ub.assign(B, 0);
    h->nlat_ub.assign(B, 0);
    TRY(set_attrs_epi<EPI_STORE>(h));
    TRY(set_attrs_epi<EPI_RESID>(h));
    TRY(set_attrs_epi<EPI_SWIGLU>(h));
    TRY(set_attrs_epi<EPI_QKV>(h));
    TRY(set_attrs_epi<EPI_LATC>(h));
    {
      int dev = 0;
      CK(cudaGetDevice(&dev));
      CK(cudaDeviceGetAttribute(&h->sm_count, cudaDevAttrMultiProcessorCount, dev));
      // split-K of small W2 grids: rows up to 64 (larger passes fill the GPU without it)
      if (F > kSegCols && F % kSegCols == 0) {
        h->seg_nmax = F / kSegCols;
        h->seg_rows = std::min(RL, 64);
        h->seg_n = d;
        TRY(dalloc(h, &h->seg_ws, (size_t)h->seg_nmax * h->seg_rows * d));
      }
    }
    if (h->tc) {
      const int KM = std::max(d, F);
      TRY(dalloc(h, &h->tc_hi, (size_t)RL * KM));
      TRY(dalloc(h, &h->tc_lo, (size_t)RL * KM));
      TRY(dalloc(h, &h->tc_rs, RL));
      CK(cudaMemset(h->tc_hi, 0, (size_t)RL * KM * 2));
      CK(cudaMemset(h->tc_lo, 0, (size_t)RL * KM * 2));
      TRY(tc_map(h, &h->tc_hi_d, h->tc_hi, d, RL, kTcBM));
      TRY(tc_map(h, &h->tc_lo_d, h->tc_lo, d, RL, kTcBM));
      TRY(tc_map(h, &h->tc_hi_f, h->tc_hi, F, RL, kTcBM));
      TRY(tc_map(h, &h->tc_lo_f, h->tc_lo, F, RL, kTcBM));
      TRY(set_tc_attrs<EPI_STORE>(h));
      TRY(set_tc_attrs<EPI_RESID>(h));
      TRY(set_tc_attrs<EPI_SWIGLU>(h));
      TRY(set_tc_attrs<EPI_QKV>(h));
    }
    TRY(set_attn_attrs<float>(h));
    TRY(set_attn_attrs<__nv_bfloat16>(h));
    TRY(mega_setup(h));
    CK(cudaDeviceSynchronize());
    return BLT_OK;
  };
  rc = run();
  if (rc != BLT_OK) {
    fprintf(stderr, "blt_dec_init: %s\n", h->err.c_str());
    blt_dec_free(h);
    return rc;
  }
  *out = h;
  return BLT_OK;
}

int blt_dec_prefill(blt_dec_t* h, int batch, const blt_rows_in* rows, float* out_logits) {
  NvtxRange nvtx_("blt_dec_prefill");
  if (!h) return BLT_ERR_INVALID_ARG;
  h->err.clear();
  if (h->state != 0) return fail(h, BLT_ERR_STATE, "a draft is waiting for verification");
  TRY(check_pending(h, rows, true));
  CallDesc cd;
  TRY(make_desc(h, batch, rows->row_offsets, rows->latent_offsets, cd));
  const int total = cd.row_off[batch];
  if (total > 0 && (!rows->bytes || !rows->row_latent)) return fail(h, BLT_ERR_INVALID_ARG, "bytes/row_latent NULL");
  refresh_bounds(h);
  return prefill_impl(h, batch, rows, out_logits, cd);
}

int blt_dec_prefill_noalloc(blt_dec_t* h, int batch, const blt_rows_in* rows, float* out_logits) {
  NvtxRange nvtx_("blt_dec_prefill_noalloc");
  if (!h) return BLT_ERR_INVALID_ARG;
  h->err.clear();
  if (h->state != 0) return fail(h, BLT_ERR_STATE, "a draft is waiting for verification");
  if (h->d > kNaMaxD || h->F > kNaMaxF || h->H > kNaMaxH || h->dh > kNaMaxDh || h->CH != kNaChunk ||
      (size_t)h->L * h->d > (size_t)kNaRows * kNaMaxD)
    return fail(h, BLT_ERR_INVALID_ARG, "model exceeds the static prefill arena (d <= %d, d_ffn <= %d, heads <= %d, head dim <= %d, "
                "attn_chunk %d, n_layers * d <= %d)", kNaMaxD, kNaMaxF, kNaMaxH, kNaMaxDh, kNaChunk, kNaRows * kNaMaxD);
  TRY(check_pending(h, rows, true));
  CallDesc cd;
  TRY(make_desc(h, batch, rows->row_offsets, rows->latent_offsets, cd));
  const int total = cd.row_off[batch];
  if (total > 0 && (!rows->bytes || !rows->row_latent)) return fail(h, BLT_ERR_INVALID_ARG, "bytes/row_latent NULL");
  refresh_bounds(h);
  for (int s = 0; s < batch; ++s)
    if (h->kv_ub[s] + cd.row_off[s + 1] - cd.row_off[s] > kNaKeys)
      return fail(h, BLT_ERR_INVALID_ARG, "sequence %d would reach %d positions > %d (static prefill arena)", s,
                  h->kv_ub[s] + cd.row_off[s + 1] - cd.row_off[s], kNaKeys);
  unsigned char* base = nullptr;
  TRY(na_arena(h, &base));
  NaSwap swap(h, base);
  if (swap.used > kNaArenaBytes) return fail(h, BLT_ERR_INVALID_ARG, "static prefill arena too small");
  return prefill_impl(h, batch, rows, out_logits, cd);
}

int blt_dec_diffuse_block(blt_dec_t* h, int batch, const blt_rows_in* pending, int k, float alpha, int max_steps,
                          uint8_t* out_block, int32_t* out_steps, float* out_logits) {
  NvtxRange nvtx_("blt_dec_diffuse_block");
  if (!h) return BLT_ERR_INVALID_ARG;
  h->err.clear();
  h->state = 0;  // a waiting draft is discarded
  TRY(check_pending(h, pending, false));
  if (k < 1 || k > h->cfg.max_block) return fail(h, BLT_ERR_INVALID_ARG, "k %d outside 1..%d", k, h->cfg.max_block);
  if (!(alpha == alpha)) return fail(h, BLT_ERR_INVALID_ARG, "alpha is NaN");
  if (!out_block) return fail(h, BLT_ERR_INVALID_ARG, "out_block is NULL");
  if (max_steps <= 0) max_steps = k;
  CallDesc cd;
  TRY(make_desc(h, batch, pending->row_offsets, pending->latent_offsets, cd));
  if (cd.row_off[batch] > 0 && (!pending->bytes || !pending->row_latent)) return fail(h, BLT_ERR_INVALID_ARG, "bytes/row_latent NULL");
  if (cd.row_off[batch] + batch * k > h->cfg.max_rows)
    return fail(h, BLT_ERR_NO_SPACE, "pass rows %d > max_rows %d", cd.row_off[batch] + batch * k, h->cfg.max_rows);
  refresh_bounds(h);
  TRY(reserve(h, cd, k, true));
  h->calls += 1;
  TRY(project_latents(h, cd, pending->new_latents, true));
  TRY(pass_begin(h));
  TRY(diffuse_passes(h, cd, pending, k, alpha, max_steps, out_logits));
  TRY(pass_end(h));
  k_finish_block<<<batch, 32, 0, h->stream>>>(h->sd, batch, k, out_block, out_steps);
  h->launches += 1;
  CK(cudaGetLastError());
  bump_bounds(h, cd, 0);
  return post_mirror(h);
}

int blt_dec_diffuse_block_eb(blt_dec_t* h, int batch, const blt_rows_in* pending, int k, float gamma, int max_steps,
                             uint8_t* out_block, int32_t* out_steps, float* out_logits) {
  NvtxRange nvtx_("blt_dec_diffuse_block_eb");
  if (!h) return BLT_ERR_INVALID_ARG;
  if (!(gamma >= 0.f) || gamma == INFINITY) {
    h->err.clear();
    return fail(h, BLT_ERR_INVALID_ARG, "gamma must be finite and >= 0");
  }
  h->eb = 1;
  const int rc = blt_dec_diffuse_block(h, batch, pending, k, gamma, max_steps, out_block, out_steps, out_logits);
  h->eb = 0;
  return rc;
}

int blt_dec_draft(blt_dec_t* h, int batch, const blt_rows_in* pending, int mode, int k, float alpha, int max_steps,
                  uint8_t* out_draft, float* out_logits) {
  NvtxRange nvtx_("blt_dec_draft");
  if (!h) return BLT_ERR_INVALID_ARG;
  if (!h->samp_on) h->err.clear();
  h->state = 0;  // a waiting draft is discarded
  h->draft_sampled = false;
  TRY(check_pending(h, pending, true));
  if (mode != BLT_DRAFT_AR && mode != BLT_DRAFT_DIFFUSION) return fail(h, BLT_ERR_INVALID_ARG, "mode %d", mode);
  if (k < 1 || k > h->cfg.max_block) return fail(h, BLT_ERR_INVALID_ARG, "k %d outside 1..%d", k, h->cfg.max_block);
  if (!out_draft) return fail(h, BLT_ERR_INVALID_ARG, "out_draft is NULL");
  if (!(alpha == alpha)) return fail(h, BLT_ERR_INVALID_ARG, "alpha is NaN");
  CallDesc cd;
  TRY(make_desc(h, batch, pending->row_offsets, pending->latent_offsets, cd));
  for (int s = 0; s < batch; ++s)
    if (cd.row_off[s + 1] - cd.row_off[s] < 1)
      return fail(h, BLT_ERR_INVALID_ARG, "sequence %d has no pending row (its prediction is y_l)", s);
  if (!pending->bytes || !pending->row_latent) return fail(h, BLT_ERR_INVALID_ARG, "bytes/row_latent NULL");
  const int rows1 = cd.row_off[batch] + (mode == BLT_DRAFT_DIFFUSION ? batch * k : 0);
  if (rows1 > h->cfg.max_rows) return fail(h, BLT_ERR_NO_SPACE, "pass rows %d > max_rows %d", rows1, h->cfg.max_rows);
  refresh_bounds(h);
  TRY(reserve(h, cd, k, true));
  h->calls += 1;
  TRY(project_latents(h, cd, pending->new_latents, true));
  TRY(pass_begin(h));
  if (mode == BLT_DRAFT_AR && use_mega(h, std::max(cd.row_off[batch], batch), batch)) {
    PlanArgs p = plan_args(h, PL_FIRST, 0);
    p.pend_bytes = pending->bytes;
    p.pend_lat = pending->row_latent;
    TRY(plan(h, p, cd));
    TRY(mega_run(h, MM_DRAFT_AR, batch, k, 0.f, k, std::max(cd.row_off[batch], batch), nullptr, out_logits, nullptr, nullptr));
  } else if (mode == BLT_DRAFT_AR) {
    int npmax = 0;
    for (int s = 0; s < batch; ++s) npmax = std::max(npmax, cd.row_off[s + 1] - cd.row_off[s]);
    const int keys_ub = max_kv_ub(h, batch) + npmax + k;
    PlanArgs p = plan_args(h, PL_FIRST, 0);
    p.pend_bytes = pending->bytes;
    p.pend_lat = pending->row_latent;
    TRY(plan(h, p, cd));
    TRY(run_pass(h, cd.row_off[batch], keys_ub, groups_bound(cd, 0), true, npmax));
    launch_draft_ar(h, batch, 0, out_logits);
    h->launches += 1;
    for (int t = 1; t < k; ++t) {
      PlanArgs pa = plan_args(h, PL_ARDRAFT, 0);
      pa.step = t;
      TRY(plan(h, pa, cd));
      TRY(run_pass(h, batch, keys_ub, batch, true, 1));
      launch_draft_ar(h, batch, t, out_logits);
      h->launches += 1;
    }
  } else {
    if (max_steps <= 0) max_steps = k;
    TRY(diffuse_passes(h, cd, pending, k, alpha, max_steps, out_logits));
  }
  TRY(pass_end(h));
  if (mode == BLT_DRAFT_DIFFUSION) k_finish_block<<<batch, 32, 0, h->stream>>>(h->sd, batch, k, out_draft, nullptr);
  else k_copy_draft<<<batch, 32, 0, h->stream>>>(h->sd, batch, k, out_draft);
  h->launches += 1;
  CK(cudaGetLastError());
  bump_bounds(h, cd, 0);
  h->state = 1;
  h->draft_k = k;
  h->draft_batch = batch;
  return post_mirror(h);
}

int blt_dec_verify_accept(blt_dec_t* h, const int32_t* draft_row_latent, const float* new_latents,
                          const int32_t* latent_offsets, int32_t* out_accepted, uint8_t* out_next, float* out_logits) {
  NvtxRange nvtx_("blt_dec_verify_accept");
  if (!h) return BLT_ERR_INVALID_ARG;
  h->err.clear();
  if (h->state != 1) return fail(h, BLT_ERR_STATE, "no draft is waiting for verification");
  if (!draft_row_latent || !out_accepted || !out_next) return fail(h, BLT_ERR_INVALID_ARG, "NULL argument");
  const int batch = h->draft_batch, k = h->draft_k;
  if (batch * k > h->cfg.max_rows) return fail(h, BLT_ERR_NO_SPACE, "pass rows %d > max_rows %d", batch * k, h->cfg.max_rows);
  CallDesc cd;
  TRY(make_desc(h, batch, nullptr, latent_offsets, cd));
  refresh_bounds(h);
  TRY(reserve(h, cd, k, false));
  h->calls += 1;
  TRY(project_latents(h, cd, new_latents, false));
  TRY(pass_begin(h));
  PlanArgs p = plan_args(h, PL_VERIFY, k);
  p.vlat = draft_row_latent;
  TRY(plan(h, p, cd));
  if (use_mega(h, batch * k, batch)) {
    TRY(mega_run(h, MM_VERIFY, batch, k, 0.f, 1, batch * k, draft_row_latent, out_logits, out_accepted, out_next));
  } else {
    TRY(run_pass(h, batch * k, max_kv_ub(h, batch) + k, batch * ((k + 31) / 32), true, k));
    if (h->samp_on)
      k_accept_sampled<<<batch, 32, 0, h->stream>>>(h->sd, batch, k, h->sa, draft_row_latent, h->logits, out_accepted, out_next,
                                                      out_logits);
    else
      k_accept<<<batch, 32, 0, h->stream>>>(h->sd, batch, k, h->pred, draft_row_latent, h->logits, out_accepted, out_next, out_logits);
    h->launches += 1;
  }
  TRY(pass_end(h));
  CK(cudaGetLastError());
  for (int s = 0; s < batch; ++s) {
    h->kv_ub[s] += k;
    h->nlat_ub[s] += cd.lat_off[s + 1] - cd.lat_off[s];
  }
  h->state = 0;
  return post_mirror(h);
}

int blt_dec_rewind(blt_dec_t* h, int batch, const int32_t* kv_len, const int32_t* n_latents) {
  NvtxRange nvtx_("blt_dec_rewind");
  if (!h) return BLT_ERR_INVALID_ARG;
  h->err.clear();
  if (batch < 1 || batch > h->cfg.max_batch) return fail(h, BLT_ERR_INVALID_ARG, "batch %d", batch);
  CallDesc cd{};
  cd.batch = batch;
  for (int s = 0; s < batch; ++s) {
    cd.row_off[s] = kv_len ? kv_len[s] : -1;
    cd.lat_off[s] = n_latents ? n_latents[s] : -1;
  }
  k_rewind<<<1, 256, 0, h->stream>>>(h->sd, cd);
  CK(cudaGetLastError());
  CK(cudaStreamSynchronize(h->stream));
  const int B = h->cfg.max_batch;
  CK(cudaMemcpy(h->mirror, h->sd.kv_len, 2 * B * 4, cudaMemcpyDeviceToHost));  // kv_len, n_lat
  for (int s = 0; s < B; ++s) {
    h->kv_ub[s] = h->mirror[s];
    h->nlat_ub[s] = h->mirror[B + s];
  }
  h->mirror_pending = false;
  h->state = 0;
  return BLT_OK;
}

int blt_dec_stats(blt_dec_t* h, blt_dec_counters* out) {
  if (!h || !out) return BLT_ERR_INVALID_ARG;
  unsigned long long c[8];
  CK(cudaStreamSynchronize(h->stream));
  TRY(drain_timing(h));
  CK(cudaMemcpy(c, h->sd.counters, sizeof c, cudaMemcpyDeviceToHost));
  out->passes = c[0];
  out->rows = c[1];
  out->prefill_rows = c[2];
  out->latents = c[3];
  out->calls = h->calls;
  out->weight_bytes = c[5];
  out->kv_read_bytes = c[6];
  out->kernel_launches = h->launches;
  out->timed_passes = (h->cfg.flags & BLT_FLAG_TIME_PASSES) ? c[0] : 0;
  out->pass_ns = h->pass_ns;
  out->persistent_calls = h->persistent_calls;
  out->prefill_kv_read_bytes = c[7];
  out->tc_gemms = h->tc_gemms;
  return BLT_OK;
}

// ---------------------------------------------------------------------------- stochastic decoding
namespace {
int sampling_on(blt_dec* h, const blt_sampling* s, int k) {
  if (!s || !s->uniforms) return fail(h, BLT_ERR_INVALID_ARG, "sampling parameters or uniforms are NULL");
  if (!(s->temperature > 0.f) || s->temperature == INFINITY) return fail(h, BLT_ERR_INVALID_ARG, "temperature must be > 0 and finite");
  if (!(s->top_p > 0.f && s->top_p <= 1.f)) return fail(h, BLT_ERR_INVALID_ARG, "top_p must be in (0, 1]");
  h->sa.temperature = s->temperature;
  h->sa.top_p = s->top_p;
  h->sa.u = s->uniforms;
  h->sa.ustride = 2 * k + 1;
  h->samp_on = true;
  return BLT_OK;
}
struct SamplingScope {  // sampling stays on for exactly one call
  blt_dec* h;
  ~SamplingScope() { h->samp_on = false; }
};
}  // namespace

int blt_dec_diffuse_block_sampled(blt_dec_t* h, int batch, const blt_rows_in* pending, int k, float threshold, int unmask,
                                  int max_steps, const blt_sampling* sampling, uint8_t* out_block, int32_t* out_steps,
                                  float* out_logits) {
  NvtxRange nvtx_("blt_dec_diffuse_block_sampled");
  if (!h) return BLT_ERR_INVALID_ARG;
  h->err.clear();
  if (unmask != BLT_UNMASK_CONFIDENCE && unmask != BLT_UNMASK_EB) return fail(h, BLT_ERR_INVALID_ARG, "unmask %d", unmask);
  TRY(sampling_on(h, sampling, k));
  SamplingScope scope{h};
  if (unmask == BLT_UNMASK_EB) return blt_dec_diffuse_block_eb(h, batch, pending, k, threshold, max_steps, out_block, out_steps, out_logits);
  return blt_dec_diffuse_block(h, batch, pending, k, threshold, max_steps, out_block, out_steps, out_logits);
}

int blt_dec_draft_sampled(blt_dec_t* h, int batch, const blt_rows_in* pending, int mode, int k, float alpha, int max_steps,
                          const blt_sampling* sampling, uint8_t* out_draft, float* out_logits) {
  NvtxRange nvtx_("blt_dec_draft_sampled");
  if (!h) return BLT_ERR_INVALID_ARG;
  h->err.clear();
  TRY(sampling_on(h, sampling, k));
  SamplingScope scope{h};
  const int rc = blt_dec_draft(h, batch, pending, mode, k, alpha, max_steps, out_draft, out_logits);
  h->draft_sampled = rc == BLT_OK;
  return rc;
}

int blt_dec_verify_sampled(blt_dec_t* h, const int32_t* draft_row_latent, const float* new_latents, const int32_t* latent_offsets,
                           const blt_sampling* sampling, int32_t* out_accepted, uint8_t* out_next, float* out_logits) {
  NvtxRange nvtx_("blt_dec_verify_sampled");
  if (!h) return BLT_ERR_INVALID_ARG;
  h->err.clear();
  if (h->state != 1 || !h->draft_sampled) return fail(h, BLT_ERR_STATE, "no drawn draft is waiting for verification");
  TRY(sampling_on(h, sampling, h->draft_k));
  SamplingScope scope{h};
  return blt_dec_verify_accept(h, draft_row_latent, new_latents, latent_offsets, out_accepted, out_next, out_logits);
}

int blt_dec_sync(blt_dec_t* h) {
  NvtxRange nvtx_("blt_dec_sync");
  if (!h) return BLT_ERR_INVALID_ARG;
  CK(cudaStreamSynchronize(h->stream));
  if (h->trace && h->trace_pending) {
    std::vector<unsigned long long> t((size_t)h->nsm * kTraceEvents);
    CK(cudaMemcpy(t.data(), h->trace, t.size() * 8, cudaMemcpyDeviceToHost));
    if (FILE* f = fopen(h->trace_path.c_str(), "ab")) {
      const int hdr[3] = {h->nsm, kTraceEvents, h->L};
      fwrite(hdr, sizeof hdr, 1, f);
      fwrite(t.data(), 8, t.size(), f);
      fclose(f);
    }
    h->trace_pending = 0;
  }
  int st = 0;
  CK(cudaMemcpy(&st, h->sd.status, 4, cudaMemcpyDeviceToHost));
  if (st != 0) {
    CK(cudaMemset(h->sd.status, 0, 4));
    return fail(h, st, "device status %d (%s)", st, st == BLT_ERR_STEP_LIMIT ? "step limit" : "device index check");
  }
  return BLT_OK;
}

const char* blt_dec_last_error(blt_dec_t* h) { return h ? h->err.c_str() : "NULL handle"; }

int blt_dec_upload(blt_dec_t* h, void* dst, const void* src, size_t n) {
  if (!h) return BLT_ERR_INVALID_ARG;
  if (n == 0) return BLT_OK;
  if (!dst || !src) return fail(h, BLT_ERR_INVALID_ARG, "blt_dec_upload: NULL pointer");
  const bool small = n <= blt_dec::kUpSmall;
  blt_dec::Bounce& b = small ? h->up[h->up_next] : h->up_large;
  if (small) h->up_next = (h->up_next + 1) % blt_dec::kUpSlots;
  if (b.done) CK(cudaEventSynchronize(b.done));  // the buffer's previous copy has run
  else CK(cudaEventCreateWithFlags(&b.done, cudaEventDisableTiming));
  if (b.cap < n) {  // small buffers: once; the large one: when a larger copy comes
    if (b.p) CK(cudaFreeHost(b.p));
    b.p = nullptr;
    b.cap = 0;
    const size_t cap = small ? blt_dec::kUpSmall : n + n / 4;
    CK(cudaHostAlloc(&b.p, cap, cudaHostAllocDefault));
    b.cap = cap;
  }
  memcpy(b.p, src, n);
  CK(cudaMemcpyAsync(dst, b.p, n, cudaMemcpyHostToDevice, h->stream));
  CK(cudaEventRecord(b.done, h->stream));
  return BLT_OK;
}

int blt_dec_download(blt_dec_t* h, void* dst, const void* src, size_t n) {
  if (!h) return BLT_ERR_INVALID_ARG;
  if (n && (!dst || !src)) return fail(h, BLT_ERR_INVALID_ARG, "blt_dec_download: NULL pointer");
  blt_dec::Bounce& b = h->down;
  if (b.cap < n) {
    if (b.p) CK(cudaFreeHost(b.p));
    b.p = nullptr;
    b.cap = 0;
    const size_t cap = std::max(n + n / 4, (size_t)1 << 16);
    CK(cudaHostAlloc(&b.p, cap, cudaHostAllocDefault));
    b.cap = cap;
  }
  if (n) CK(cudaMemcpyAsync(b.p, src, n, cudaMemcpyDeviceToHost, h->stream));
  CK(cudaStreamSynchronize(h->stream));
  if (n) memcpy(dst, b.p, n);
  return BLT_OK;
}

void blt_dec_free(blt_dec_t* h) {
  if (!h) return;
  if (h->stream) cudaStreamSynchronize(h->stream);
  for (int i = 0; i <= blt_dec::kUpSlots; ++i) {
    blt_dec::Bounce& b = i < blt_dec::kUpSlots ? h->up[i] : h->up_large;
    if (b.p) cudaFreeHost(b.p);
    if (b.done) cudaEventDestroy(b.done);
  }
  if (h->down.p) cudaFreeHost(h->down.p);
  for (void* p : h->allocs) cudaFree(p);
  if (h->mirror) cudaFreeHost(h->mirror);
  if (h->mirror_ev) cudaEventDestroy(h->mirror_ev);
  for (cudaEvent_t e : h->tev) cudaEventDestroy(e);
  if (h->own_stream && h->stream) cudaStreamDestroy(h->stream);
  delete h;
}

}  // extern "C"
