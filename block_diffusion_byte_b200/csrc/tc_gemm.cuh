// Projections of decoder passes with many rows on the 5th-generation tensor
// cores (tcgen05, accumulator in tensor memory, operands staged by TMA).
//
// Fast-BLT (block diffusion): with batch x block rows per pass the decoder's
// projections become dense contractions (the pages' decoder layer: QKV, O and
// SwiGLU projections over all rows of a pass, "BLT-D 추론"); at 128 rows and more
// the legacy mma.sync GEMV of kernels.cuh is compute-bound, so these passes run
// here.  Same math as k_gemm: the activation row times the gain, split into bf16
// hi + lo (both multiplied by the bf16 weights, fp32 accumulate), times the
// row's RMS scale, then the same fused epilogues (gemm_epilogue).  The order of
// the fp32 sums differs from k_gemm's canonical order, so results agree to
// rounding, not bit for bit.
//
// Tile: 128 activation rows (TMEM lanes) x BN output features; K in steps of
// 64 (one 128-byte swizzle atom of bf16).  Thread 0 issues the TMA loads
// (no multicast), thread 32 the MMAs (cta_group::1, kind::f16, bf16 x bf16 ->
// fp32); all four warps read the accumulator back (tcgen05.ld 32x32b) into
// shared memory and then run the epilogue row by row, a warp on consecutive
// columns.  Every wait is bounded in wall time.
#pragma once

#include <cuda.h>

#include "kernels.cuh"

namespace bltdec {

constexpr int kTcBM = 128;     // activation rows per tile
constexpr int kTcBK = 64;      // K per stage (bf16: 128 bytes, the swizzle atom)
constexpr int kTcStages = 4;   // smem pipeline depth
constexpr int kTcMinRows = 128;

__host__ __device__ constexpr unsigned tc_stage_bytes(int bn) { return 2u * kTcBM * kTcBK * 2u + (unsigned)bn * kTcBK * 2u; }
__host__ __device__ constexpr size_t tc_smem_bytes(int bn) { return (size_t)kTcStages * tc_stage_bytes(bn) + 1024; }

// ---------------------------------------------------------------------------- activation prep
// Row `row` of X times the gain -> bf16 hi and lo planes ([rows][K], row
// stride K), and the row's scale 1 / sqrt(mean(x^2) + eps) (1 without a gain).
// K a multiple of 4; X rows 16-byte aligned.
__global__ void __launch_bounds__(256) k_tc_prep(const float* __restrict__ X, int ldx, int K, const float* __restrict__ gain,
                                                 float eps, const int* n_rows, int rows_cap, __nv_bfloat16* __restrict__ hi,
                                                 __nv_bfloat16* __restrict__ lo, float* __restrict__ rs) {
  const int row = blockIdx.x;
  const int nrows = n_rows ? *n_rows : rows_cap;
  if (row >= nrows) return;  // its outputs are never stored
  const float* x = X + (size_t)row * ldx;
  float ss = 0.f;
  for (int c = threadIdx.x * 4; c < K; c += 256 * 4) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(x + c));
    float4 g = make_float4(1.f, 1.f, 1.f, 1.f);
    if (gain) g = __ldg(reinterpret_cast<const float4*>(gain + c));
    ss = fmaf(v.x, v.x, ss);
    ss = fmaf(v.y, v.y, ss);
    ss = fmaf(v.z, v.z, ss);
    ss = fmaf(v.w, v.w, ss);
    uint32_t h0, l0, h1, l1;
    split2(v.x * g.x, v.y * g.y, h0, l0);
    split2(v.z * g.z, v.w * g.w, h1, l1);
    *reinterpret_cast<uint2*>(hi + (size_t)row * K + c) = make_uint2(h0, h1);
    *reinterpret_cast<uint2*>(lo + (size_t)row * K + c) = make_uint2(l0, l1);
  }
  __shared__ float red[8];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += red[w];
    rs[row] = gain ? 1.0f / sqrtf(t / (float)K + eps) : 1.0f;
  }
}

// ---------------------------------------------------------------------------- tcgen05 / TMA primitives
__device__ __forceinline__ uint32_t tc_smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Shared-memory matrix descriptor: K-major tile of 64 bf16 per row (128-byte
// rows, 128-byte swizzle as TMA writes it), 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t tc_desc_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address, 16-byte units
  d |= (uint64_t)1 << 16;                             // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;                   // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;                             // descriptor version (tcgen05)
  d |= (uint64_t)2 << 61;                             // 128-byte swizzle
  return d;
}
// Instruction descriptor: bf16 x bf16 -> fp32, A and B K-major, M = 128, N = bn.
__host__ __device__ constexpr uint32_t tc_idesc(int bn) {
  return (1u << 4)                        // D format fp32
         | (1u << 7)                      // A format bf16
         | (1u << 10)                     // B format bf16
         | ((uint32_t)(bn >> 3) << 17)    // N / 8
         | ((uint32_t)(kTcBM >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void tc_mbar_init(uint64_t* b, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(tc_smem_u32(b)), "r"(count));
}
__device__ __forceinline__ void tc_expect_tx(uint64_t* b, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(tc_smem_u32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool tc_mbar_try(uint64_t* b, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(tc_smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long tc_now() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for phase `parity` of barrier b; false once wait_ns of wall time have passed.
__device__ __forceinline__ bool tc_wait(uint64_t* b, unsigned parity, unsigned long long wait_ns) {
  if (tc_mbar_try(b, parity)) return true;
  const unsigned long long t0 = tc_now();
  while (!tc_mbar_try(b, parity))
    if (tc_now() - t0 > wait_ns) return false;
  return true;
}
// 2-D tiled TMA load (no multicast): box at (x = inner element, y = row).
__device__ __forceinline__ void tc_tma_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
          tc_smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(tc_smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}
// Arrive on `bar` once every MMA this thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(tc_smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
// 32 consecutive fp32 columns of this warp's 32 TMEM lanes (one lane per thread).
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]),
        "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
        "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]),
        "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}

// ---------------------------------------------------------------------------- the GEMM
// out-tile (blockIdx.y: 128 rows, blockIdx.x: BN features) of
// X[rows][K] . W[N][K]^T through gemm_epilogue<EPI>.  ta_hi / ta_lo: the
// prepared activation planes (box 64 x 128), tb: the weights, row-major bf16
// in the packed row order of kernels.cuh (box 64 x BN).  rs: row scales.
template <int BN, int EPI>
__global__ void __launch_bounds__(128, 1)
    k_tc_gemm(const __grid_constant__ CUtensorMap ta_hi, const __grid_constant__ CUtensorMap ta_lo,
              const __grid_constant__ CUtensorMap tb, GemmArgs a, const float* __restrict__ rs, unsigned long long wait_ns) {
  static_assert(BN == 32 || BN == 64 || BN == 128, "TMEM columns: a power of two >= 32");
  constexpr unsigned A_BYTES = kTcBM * kTcBK * 2;
  constexpr unsigned STAGE = tc_stage_bytes(BN);
  extern __shared__ unsigned char tc_smem_raw[];
  __shared__ uint64_t full[kTcStages], empty[kTcStages], done;
  __shared__ uint32_t tmem_base;

  const int nrows = a.n_rows ? *a.n_rows : a.rows_host;
  const int row0 = blockIdx.y * kTcBM;
  if (row0 >= nrows) return;
  const int n0 = blockIdx.x * BN;
  const int nkb = a.K / kTcBK;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~(uintptr_t)1023);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(tc_smem_u32(&tmem_base)), "r"(BN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < kTcStages; ++s) {
      tc_mbar_init(full + s, 1);
      tc_mbar_init(empty + s, 1);
    }
    tc_mbar_init(&done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  bool ok = true;

  if (threadIdx.x == 0) {  // TMA producer
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % kTcStages;
      if (kb >= kTcStages && !tc_wait(empty + s, ((kb / kTcStages) - 1) & 1, wait_ns)) {
        ok = false;
        break;
      }
      unsigned char* st = smem + (size_t)s * STAGE;
      tc_expect_tx(full + s, STAGE);
      tc_tma_2d(st, &ta_hi, kb * kTcBK, row0, full + s);
      tc_tma_2d(st + A_BYTES, &ta_lo, kb * kTcBK, row0, full + s);
      tc_tma_2d(st + 2 * A_BYTES, &tb, kb * kTcBK, n0, full + s);
    }
  } else if (threadIdx.x == 32) {  // MMA issuer
    constexpr uint32_t idesc = tc_idesc(BN);
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % kTcStages;
      if (!tc_wait(full + s, (kb / kTcStages) & 1, wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t st = tc_smem_u32(smem + (size_t)s * STAGE);
      const uint64_t dh = tc_desc_sw128(st), dl = tc_desc_sw128(st + A_BYTES), db = tc_desc_sw128(st + 2 * A_BYTES);
#pragma unroll
      for (int kk = 0; kk < kTcBK / 16; ++kk) {  // k16 steps: +32 bytes inside the swizzle atom
        tc_mma(tmem, dh + 2 * kk, db + 2 * kk, idesc, kb > 0 || kk > 0);
        tc_mma(tmem, dl + 2 * kk, db + 2 * kk, idesc, true);
      }
      tc_commit(empty + s);  // the stage is free once these MMAs have read it
    }
    if (ok) tc_commit(&done);  // on a failed wait the others' waits run out too
  }
  __syncwarp();
  if (!tc_wait(&done, 0, wait_ns)) ok = false;
  tc_fence_after();
  // Accumulator -> shared memory (times the row scale), [128][BN + 1] over the stage buffers:
  // every copy and MMA has completed.  Thread = row here; the epilogue then walks rows with
  // a warp on consecutive columns, so its stores are coalesced.
  constexpr int TS = BN + 1;
  float* tile = reinterpret_cast<float*>(smem);
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // generic writes after the tensor cores' reads
  const int rl = warp * 32 + lane;
  const float scale = (row0 + rl < nrows) ? __ldcg(rs + row0 + rl) : 0.f;
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 32) {
    uint32_t v[32];
    tc_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) tile[rl * TS + c0 + j] = __uint_as_float(v[j]) * scale;
  }
  tc_fence_before();
  const bool all_ok = __syncthreads_and(ok) != 0;
  if (all_ok) {
    const int nr = min(kTcBM, nrows - row0);
    const int grp = lane >> 3, r16 = lane & 7;  // lane: pair (r16, r16 + 8) of 16-column group grp
#pragma unroll 1
    for (int r = warp; r < nr; r += 4)
#pragma unroll
      for (int g0 = 0; g0 < BN / 16; g0 += 4) {
        const int g = g0 + grp;
        if (g < BN / 16) {
          const float* tr = tile + r * TS + 16 * g + r16;
          gemm_epilogue<EPI>(a, (n0 >> 4) + g, r16, row0 + r, tr[0], tr[8]);
        }
      }
  }
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(BN));
  if (!all_ok && threadIdx.x == 0) set_status(a.status, kErrDevice);
}

}  // namespace bltdec
