// W8A8 product with per-token x per-channel scales on the sm_100a tensor
// cores (tcgen05), the consumer of the quantizer's codes.
//
// aclnnQuantBatchMatmulInplaceAdd, "计算公式" (T-T form): the quantized product
// sum_k x1[m,k] * x2[k,n] is multiplied by (scale1 * scale2) and added to y.
// Here scale1 is per row of x1 (per token, as dq_dynamic_quant produces it)
// and scale2 per output column (per channel of the weights):
//   acc[m,n] = sum_k a[m,k] * b[n,k]                      (exact, int32)
//   out[m,n] = float(acc) * (a_scale[m] * b_scale[n])  (+ out[m,n])
// each binary32 operation rounded once in that order, then narrowed.
//
// Tensor-core path (K a multiple of 16, 16-byte aligned operands; any M, N):
// one CTA per 128 x BN output tile, 6 warps, BN = 256 unless a 128-wide last
// tile wastes less. Tiles past M, N or K are zero-filled by the loads and
// masked in the epilogue.
//   warp 0      TMA producer: 128-byte K slices of 128 rows of A and BN rows
//               of B (K-major, 128-byte swizzle) into a shared-memory ring.
//   warp 1      allocates BN TMEM columns (the int32 accumulator, row m in
//               lane m); one lane issues tcgen05.mma.kind::i8 (M=128, N=BN,
//               K=32, four per stage) and releases each stage with
//               tcgen05.commit, then commits the accumulator.
//   warps 2-5   epilogue: the tile's column scales staged in shared memory,
//               tcgen05.ld of their 32-lane quarter, 32 columns at a time,
//               scales, optional accumulation, narrowing, 16-byte stores.
// The ring holds 96 KB (2 stages of 48 KB at BN = 256, 3 of 32 KB at 128),
// so two CTAs share an SM (and its 512 TMEM columns) and one's epilogue
// overlaps the other's main loop. The 256-wide tile reads 48 KB of operands
// per 2^22 multiply-adds instead of 64 KB: on 4096^3, 58.6 us against 65.4.
// Every mbarrier wait is bounded; the MMA lane always issues the final
// commit, so teardown never frees TMEM under MMAs in flight. A tile whose
// sum is incomplete (the epilogue's wait ran out, or the MMA lane gave up on
// a stage and flagged it) is written as NaN, and the producer waits
// (bounded) for its copies in flight before the CTA exits.
// K not a multiple of 16, or unaligned operands: a CUDA-core kernel with the
// same arithmetic.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "dq.h"
#include "tma_pipeline.cuh"

namespace {

// Output tile kBM x BN (BN = 128 or 256 columns), K in steps of kBK bytes =
// one 128-byte swizzle row.
constexpr int kBM = 128, kBK = 128;
#ifndef DQ_W8A8_BN
#define DQ_W8A8_BN 256  // widest tile the dispatcher may use (4096^3: 58.6 us at 256, 65.4 at 128)
#endif
#ifndef DQ_W8A8_STAGES_128
#define DQ_W8A8_STAGES_128 3  // 96 KB of ring: two CTAs share an SM, one's epilogue overlapping the other's MMAs
#endif
#ifndef DQ_W8A8_STAGES_256
#define DQ_W8A8_STAGES_256 2  // 96 KB of ring for 128 x 256 tiles: again two CTAs per SM
#endif
constexpr uint32_t kTileABytes = kBM * kBK;  // 16 KB
constexpr int kThreads = 192;

// Instruction descriptor of tcgen05.mma kind::i8 for an M = 128 x N tile:
// int32 accumulator (format 2), signed A and B (format 1), both K-major,
// N / 8 and M / 16.
constexpr uint32_t i8_idesc(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
}

template <int BN, int STAGES>
struct TileConfig {
  static constexpr uint32_t kTileBBytes = BN * kBK;
  static constexpr uint32_t kStageBytes = kTileABytes + kTileBBytes;
  static constexpr uint32_t kTmemCols = BN;  // one int32 accumulator column per output column
  // slack for 1024-byte alignment, ring, barriers, column scales
  static constexpr size_t kSmemBytes = 1024 + STAGES * kStageBytes + 256 + BN * 4;
  static constexpr uint32_t kIdesc = i8_idesc(BN);
};

struct W8A8Args {
  const int8_t* a;
  const int8_t* b;
  const float* a_scale;
  const float* b_scale;
  void* out;
  int64_t m, n, k;
  int out_kind;    // 0 f32, 1 f16, 2 bf16
  int accumulate;  // out (f32) += product
  int vec_out;     // out is 16-byte aligned: whole-row-chunk vector stores
};

// Quiet NaN in the output type: the mark of a tile whose accumulator never
// became ready (a bounded wait ran out).
__device__ __forceinline__ void store_nan(const W8A8Args& a, int64_t e) {
  if (a.out_kind == 0) {
    static_cast<float*>(a.out)[e] = __int_as_float(0x7fc00000);
  } else {
    static_cast<uint16_t*>(a.out)[e] = a.out_kind == 1 ? uint16_t(0x7e00) : uint16_t(0x7fc0);
  }
}

__device__ __forceinline__ void store_out(const W8A8Args& a, int64_t e, float t) {
  if (a.out_kind == 0) {
    float* o = static_cast<float*>(a.out);
    o[e] = a.accumulate ? __fadd_rn(t, o[e]) : t;
  } else if (a.out_kind == 1) {
    static_cast<__half*>(a.out)[e] = __float2half_rn(t);
  } else {
    static_cast<__nv_bfloat16*>(a.out)[e] = __float2bfloat16_rn(t);
  }
}

// Epilogue of one 32-column chunk of one output row: out = float(acc) *
// (a_scale[row] * b_scale[col]) (+ out), narrowed, with 16-byte stores when
// the whole chunk is in range and rows start 16-byte aligned. `cs` holds the
// chunk's 32 column scales.
__device__ __forceinline__ void epilogue_chunk(const W8A8Args& a, int64_t row, int64_t c0, const uint32_t (&r)[32],
                                               float sa_row, const float* cs) {
  float t[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float scales = __fmul_rn(sa_row, cs[j]);
    t[j] = __fmul_rn(__int2float_rn(static_cast<int>(r[j])), scales);
  }
  const int64_t e0 = row * a.n + c0;  // 32 consecutive outputs of this row
  if (a.vec_out && c0 + 32 <= a.n) {
    if (a.out_kind == 0) {
      float4* o = reinterpret_cast<float4*>(static_cast<float*>(a.out) + e0);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float4 v = make_float4(t[4 * q], t[4 * q + 1], t[4 * q + 2], t[4 * q + 3]);
        if (a.accumulate) {
          const float4 y = o[q];
          v = make_float4(__fadd_rn(v.x, y.x), __fadd_rn(v.y, y.y), __fadd_rn(v.z, y.z), __fadd_rn(v.w, y.w));
        }
        o[q] = v;
      }
    } else {
      uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + e0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float x0 = t[8 * q + 2 * h], x1 = t[8 * q + 2 * h + 1];
          if (a.out_kind == 1) {
            const __half2 p2 = __floats2half2_rn(x0, x1);
            w[h] = *reinterpret_cast<const uint32_t*>(&p2);
          } else {
            const __nv_bfloat162 p2 = __floats2bfloat162_rn(x0, x1);
            w[h] = *reinterpret_cast<const uint32_t*>(&p2);
          }
        }
        o[q] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (c0 + j < a.n) store_out(a, e0 + j, t[j]);
    }
  }
}

// ---------------------------------------------------------------- tcgen05 helpers

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major tile in the 128-byte swizzle
// layout: rows of 128 bytes, groups of 8 rows 1024 bytes apart (stride byte
// offset 1024; the leading byte offset is 1 for swizzled K-major tiles),
// descriptor version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc_k_sw128(const void* tile) {
  const uint64_t start = (dq::smem_addr(tile) >> 4) & 0x3FFFu;
  return start | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// The same for the 64-byte swizzle layout: rows of 64 bytes, groups of 8
// rows 512 bytes apart, layout type 4.
__device__ __forceinline__ uint64_t smem_desc_k_sw64(const void* tile) {
  const uint64_t start = (dq::smem_addr(tile) >> 4) & 0x3FFFu;
  return start | (uint64_t(1) << 16) | (uint64_t(512 >> 4) << 32) | (uint64_t(1) << 46) | (uint64_t(4) << 61);
}

__device__ __forceinline__ void tc_mma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(dq::smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dq::smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(dq::smem_addr(bar))
      : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tc_ld_32cols(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- bounded waits

__device__ __forceinline__ bool wait_or_abort_for(uint64_t* bar, uint32_t parity, const volatile uint32_t* abort,
                                                  uint64_t limit_ns) {
  const uint32_t addr = dq::smem_addr(bar);
  if (dq::mbar_try_wait(addr, parity)) return true;
  const uint64_t t0 = dq::global_ns();
  while (true) {
    if (dq::mbar_try_wait(addr, parity)) return true;
    if (*abort != 0u || dq::global_ns() - t0 > limit_ns) return false;
  }
}

// Wait for an accumulator that the MMA lane is still building: gives up only
// after kWaitLimitNs without the lane's stage counter `progress` moving (or
// on the abort flag), so a long K loop that keeps moving is never cut off,
// while a stuck one ends within the limit.
__device__ __forceinline__ bool wait_while_progress(uint64_t* bar, uint32_t parity, const volatile uint32_t* abort,
                                                    const volatile uint32_t* progress) {
  const uint32_t addr = dq::smem_addr(bar);
  if (dq::mbar_try_wait(addr, parity)) return true;
  uint64_t t0 = dq::global_ns();
  uint32_t seen = *progress;
  while (true) {
    if (dq::mbar_try_wait(addr, parity)) return true;
    if (abort != nullptr && *abort != 0u) return false;
    const uint32_t now_seen = *progress;
    const uint64_t now = dq::global_ns();
    if (now_seen != seen) {
      seen = now_seen;
      t0 = now;
    } else if (now - t0 > dq::kWaitLimitNs) {
      return false;
    }
  }
}

// ---------------------------------------------------------------- kernels

template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
w8a8_gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                    const W8A8Args a) {
  using Cfg = TileConfig<BN, STAGES>;
  constexpr int kStages = STAGES;
  constexpr int kBN = BN;
  constexpr uint32_t kTmemCols = Cfg::kTmemCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sa = smem;                             // kStages x 16 KB (A tiles)
  uint8_t* sb = smem + kStages * kTileABytes;     // kStages x BN * 128 bytes (B tiles)
  uint64_t* full = reinterpret_cast<uint64_t*>(sb + kStages * Cfg::kTileBBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_ready = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_ready + 1);
  volatile uint32_t* mma_failed = tmem_slot + 1;  // set when the MMA lane gave up on a stage
  volatile uint32_t* mma_progress = tmem_slot + 2;  // stages the MMA lane has consumed
  float* col_scale = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 256);  // the tile's b_scale

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kBM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kBN;
  const int ktiles = static_cast<int>((a.k + kBK - 1) / kBK);  // the last slice is zero-filled past k

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      dq::mbar_init(full + s, 1);
      dq::mbar_init(empty + s, 1);
    }
    dq::mbar_init(acc_ready, 1);
    *mma_failed = 0u;
    *mma_progress = 0u;
    dq::fence_mbarrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dq::smem_addr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // launched as a programmatic dependent: the codes may come from the
  // previous kernel, so no global memory is read before this
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    if (lane == 0) {  // producer
      int issued = 0;
      for (int kt = 0; kt < ktiles; ++kt, ++issued) {
        const int s = kt % kStages;
        const uint32_t ph = static_cast<uint32_t>(kt / kStages) & 1u;
        if (!dq::mbar_wait_parity(empty + s, ph ^ 1u)) break;
#if defined(DQ_TEST_SKIP_W8A8_TILE_M) && defined(DQ_TEST_SKIP_W8A8_KTILE)
        // test builds only: leave one operand stage of one tile out, so that
        // the MMA lane's bounded wait runs out and the failure path runs
        if (blockIdx.y == DQ_TEST_SKIP_W8A8_TILE_M && blockIdx.x == 0 && kt == DQ_TEST_SKIP_W8A8_KTILE) continue;
#endif
        dq::mbar_arrive_expect_tx(full + s, Cfg::kStageBytes);
        tma_load_2d(sa + s * kTileABytes, &map_a, kt * kBK, static_cast<int>(m0), full + s);
        tma_load_2d(sb + s * Cfg::kTileBBytes, &map_b, kt * kBK, static_cast<int>(n0), full + s);
      }
      // no copy may still be landing in this CTA's shared memory when it
      // exits: wait (bounded) for the last copy of every stage. Normally they
      // have long landed; after a timed-out wait elsewhere this drains them.
      for (int kt = issued > kStages ? issued - kStages : 0; kt < issued; ++kt) {
        dq::mbar_wait_parity(full + kt % kStages, static_cast<uint32_t>(kt / kStages) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      for (int kt = 0; kt < ktiles; ++kt) {
        const int s = kt % kStages;
        const uint32_t ph = static_cast<uint32_t>(kt / kStages) & 1u;
        if (!dq::mbar_wait_parity(full + s, ph)) {
          // the sum will miss this stage: tell the epilogue before the commit
          *mma_failed = 1u;
          __threadfence_block();
          break;
        }
        tc_fence_after();
        const uint64_t ad = smem_desc_k_sw128(sa + s * kTileABytes);
        const uint64_t bd = smem_desc_k_sw128(sb + s * Cfg::kTileBBytes);
#pragma unroll
        for (int kk = 0; kk < kBK / 32; ++kk) {
          // +32 bytes along K = +2 in the descriptor's 16-byte address units
          tc_mma_i8(tmem, ad + 2 * kk, bd + 2 * kk, Cfg::kIdesc, (kt | kk) != 0 ? 1u : 0u);
        }
        tc_commit(empty + s);  // the stage is free once these MMAs have read it
        *mma_progress = static_cast<uint32_t>(kt + 1);
      }
      tc_commit(acc_ready);  // every MMA issued above is complete when this arrives
      // this warp frees the TMEM below: it sees the MMAs complete itself, so
      // the accumulator is never released under MMAs still in flight (even
      // when the epilogue's wait has run out)
      dq::mbar_wait_parity(acc_ready, 0);
    }
  } else {  // epilogue: warps 2..5 cover TMEM lane quarters (warp % 4)
    // the tile's column scales, staged once by the 128 epilogue threads
#pragma unroll
    for (int j = threadIdx.x - 64; j < kBN; j += 128) col_scale[j] = n0 + j < a.n ? a.b_scale[n0 + j] : 0.0f;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    // the MMA lane may take up to one wait limit per stage: the epilogue
    // gives up only when the lane has stopped moving for that long
    const bool ready = wait_while_progress(acc_ready, 0, nullptr, mma_progress) && *mma_failed == 0u;
    tc_fence_after();
    const int quarter = warp & 3;
    const int64_t row = m0 + 32 * quarter + lane;
    const bool row_ok = row < a.m;  // rows past m (zero-filled operands) are not stored
    const float sa_row = row_ok ? a.a_scale[row] : 0.0f;
#pragma unroll 1
    for (int c = 0; c < kBN / 32; ++c) {
      const int64_t c0 = n0 + 32 * c;
      if (c0 >= a.n) break;  // the same for every lane: the collective loads below stay warp-uniform
      uint32_t r[32];
      tc_ld_32cols(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + static_cast<uint32_t>(32 * c), r);
      if (!row_ok) continue;
      if (!ready) {  // the accumulator never became ready: NaN marks the tile
        for (int j = 0; j < 32; ++j) {
          if (c0 + j < a.n) store_nan(a, row * a.n + c0 + j);
        }
        continue;
      }
      epilogue_chunk(a, row, c0, r, sa_row, col_scale + 32 * c);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ---------------------------------------------------------------- persistent kernel

// One CTA per SM walks a list of output tiles: 128 x 256 tiles first, then the
// last r of them split into two 128 x 128 tiles each, when that evens out the
// SMs (every SM gets q wide tiles, 2r <= SMs of them one narrow tile: the
// last wave is half as long). The ring holds 192 KB of K slices of kPBK bytes
// (4 stages of 48 KB at 128 bytes, 8 of 24 KB at 64); the int32 accumulator is
// double-buffered in TMEM (2 x 256 columns), so the epilogue of one tile
// overlaps the MMAs of the next.
#ifndef DQ_W8A8_PBK
#define DQ_W8A8_PBK 128
#endif
constexpr int kPBK = DQ_W8A8_PBK;  // K slice per stage: 128 (128-byte swizzle) or 64 (64-byte swizzle)
static_assert(kPBK == 128 || kPBK == 64, "K slice of 64 or 128 bytes");
#ifndef DQ_W8A8_PSTAGES
#define DQ_W8A8_PSTAGES (kPBK == 128 ? 4 : 8)
#endif
constexpr int kPStages = DQ_W8A8_PSTAGES;
constexpr uint32_t kPTileABytes = kBM * kPBK;                     // 16 KB at 128
constexpr uint32_t kPTileBBytes = 256 * kPBK;                     // 32 KB at 128 (a narrow tile uses half)
constexpr uint32_t kPStageBytes = kPTileABytes + kPTileBBytes;   // 48 KB at 128
constexpr uint32_t kPTmemCols = 512;
// ring, barriers and flags (256 B), two buffers of 256 column scales
constexpr size_t kPSmemBytes = 1024 + kPStages * kPStageBytes + 256 + 2 * 256 * 4;

__device__ __forceinline__ uint64_t smem_desc_k_p(const void* tile) {
  return kPBK == 128 ? smem_desc_k_sw128(tile) : smem_desc_k_sw64(tile);
}
constexpr uint32_t kIdescN256 = i8_idesc(256);
constexpr uint32_t kIdescN128 = i8_idesc(128);

struct PersistSched {
  int64_t n_tiles;  // 256-wide column tiles
  int64_t wide;     // list items that are whole 128 x 256 tiles
  int64_t items;    // wide + 2 * (tiles split in two)
};

__device__ __forceinline__ void decode_item(const PersistSched& ps, int64_t item, int64_t& m0, int64_t& n0,
                                            bool& wide) {
  int64_t t, half = 0;
  if (item < ps.wide) {
    t = item;
    wide = true;
  } else {
    t = ps.wide + (item - ps.wide) / 2;
    half = (item - ps.wide) & 1;
    wide = false;
  }
  m0 = (t / ps.n_tiles) * kBM;
  n0 = (t % ps.n_tiles) * 256 + half * 128;
}

__global__ void __launch_bounds__(kThreads, 1)
w8a8_gemm_persistent_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b256,
                            const __grid_constant__ CUtensorMap map_b128, const W8A8Args a, const PersistSched ps) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sa = smem;                                   // kPStages x kPTileABytes (A tiles)
  uint8_t* sb = smem + kPStages * kPTileABytes;         // kPStages x kPTileBBytes (B tiles)
  uint64_t* full = reinterpret_cast<uint64_t*>(sb + kPStages * kPTileBBytes);
  uint64_t* empty = full + kPStages;
  uint64_t* acc_full = empty + kPStages;   // [2]: the accumulator holds a finished tile
  uint64_t* acc_empty = acc_full + 2;      // [2]: the epilogue has read it out
  uint64_t* mma_done = acc_empty + 2;      // every MMA this CTA issued has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* mma_progress = tmem_slot + 2;  // stages the MMA lane has consumed
  float* col_scale = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 256);  // [2][256]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ktiles = static_cast<int>((a.k + kPBK - 1) / kPBK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      dq::mbar_init(full + s, 1);
      dq::mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      dq::mbar_init(acc_full + b, 1);
      dq::mbar_init(acc_empty + b, 4);  // one arrival per epilogue warp
    }
    dq::mbar_init(mma_done, 1);
    *abort_flag = 0u;
    *mma_progress = 0u;
    dq::fence_mbarrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dq::smem_addr(tmem_slot)),
                 "r"(kPTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // launched as a programmatic dependent: the codes may come from the
  // previous kernel, so no global memory is read before this
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    if (lane == 0) {  // producer
      uint32_t slice = 0;
      bool ok = true;
      for (int64_t item = blockIdx.x; ok && item < ps.items; item += gridDim.x) {
        int64_t m0, n0;
        bool wide;
        decode_item(ps, item, m0, n0, wide);
        for (int kt = 0; kt < ktiles; ++kt, ++slice) {
          const int s = static_cast<int>(slice % kPStages);
          const uint32_t ph = (slice / kPStages) & 1u;
          if (!wait_or_abort_for(empty + s, ph ^ 1u, abort_flag, dq::kWaitLimitNs)) {
            *abort_flag = 1u;
            ok = false;
            break;
          }
#if defined(DQ_TEST_SKIP_W8A8_TILE_M) && defined(DQ_TEST_SKIP_W8A8_KTILE)
          // test builds only: leave one operand stage of one tile out, so that
          // the MMA lane's bounded wait runs out and the failure path runs
          if (m0 == int64_t(kBM) * DQ_TEST_SKIP_W8A8_TILE_M && n0 == 0 && kt == DQ_TEST_SKIP_W8A8_KTILE) continue;
#endif
          dq::mbar_arrive_expect_tx(full + s, kPTileABytes + (wide ? kPTileBBytes : kPTileBBytes / 2));
          tma_load_2d(sa + s * kPTileABytes, &map_a, kt * kPBK, static_cast<int>(m0), full + s);
          tma_load_2d(sb + s * kPTileBBytes, wide ? &map_b256 : &map_b128, kt * kPBK, static_cast<int>(n0), full + s);
        }
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (uint32_t j = slice > kPStages ? slice - kPStages : 0; j < slice; ++j) {
        dq::mbar_wait_parity(full + j % kPStages, (j / kPStages) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      uint32_t slice = 0;
      bool ok = true;
      int i = 0;
      for (int64_t item = blockIdx.x; ok && item < ps.items; item += gridDim.x, ++i) {
        int64_t m0, n0;
        bool wide;
        decode_item(ps, item, m0, n0, wide);
        const int acc = i & 1;
        if (!wait_or_abort_for(acc_empty + acc, ((i >> 1) & 1) ^ 1u, abort_flag, dq::kWaitLimitNs)) {
          *abort_flag = 1u;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(acc * 256);
        const uint32_t idesc = wide ? kIdescN256 : kIdescN128;
        for (int kt = 0; kt < ktiles; ++kt, ++slice) {
          const int s = static_cast<int>(slice % kPStages);
          const uint32_t ph = (slice / kPStages) & 1u;
          if (!wait_or_abort_for(full + s, ph, abort_flag, dq::kWaitLimitNs)) {
            *abort_flag = 1u;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = smem_desc_k_p(sa + s * kPTileABytes);
          const uint64_t bd = smem_desc_k_p(sb + s * kPTileBBytes);
#pragma unroll
          for (int kk = 0; kk < kPBK / 32; ++kk) {
            tc_mma_i8(d, ad + 2 * kk, bd + 2 * kk, idesc, (kt | kk) != 0 ? 1u : 0u);
          }
          tc_commit(empty + s);
          *mma_progress = slice + 1;
        }
        if (ok) tc_commit(acc_full + acc);
      }
      // this warp frees the TMEM below: it sees every MMA it issued complete
      tc_commit(mma_done);
      dq::mbar_wait_parity(mma_done, 0);
    }
  } else {  // epilogue: warps 2..5 cover TMEM lane quarters (warp % 4)
    const int quarter = warp & 3;
    const int et = threadIdx.x - 64;
    bool dead = false;
    int i = 0;
    for (int64_t item = blockIdx.x; item < ps.items; item += gridDim.x, ++i) {
      int64_t m0, n0;
      bool wide;
      decode_item(ps, item, m0, n0, wide);
      const int bn = wide ? 256 : 128;
      const int acc = i & 1;
      float* cs = col_scale + acc * 256;
      for (int j = et; j < bn; j += 128) cs[j] = n0 + j < a.n ? a.b_scale[n0 + j] : 0.0f;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (!dead) dead = !wait_while_progress(acc_full + acc, (i >> 1) & 1, abort_flag, mma_progress);
      // lanes can see a wait's deadline differently: the warp agrees, so the
      // collective TMEM loads below are taken by all of its lanes or none
      dead = __any_sync(0xffffffffu, dead);
      tc_fence_after();
      const int64_t row = m0 + 32 * quarter + lane;
      const bool row_ok = row < a.m;
      const float sa_row = row_ok ? a.a_scale[row] : 0.0f;
#pragma unroll 1
      for (int c = 0; c < bn / 32; ++c) {
        const int64_t c0 = n0 + 32 * c;
        if (c0 >= a.n) break;  // warp-uniform
        if (dead) {  // a wait ran out in this CTA: NaN marks this and its remaining tiles
          if (row_ok) {
            for (int j = 0; j < 32; ++j) {
              if (c0 + j < a.n) store_nan(a, row * a.n + c0 + j);
            }
          }
          continue;
        }
        uint32_t r[32];
        tc_ld_32cols(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + static_cast<uint32_t>(acc * 256 + 32 * c),
                     r);
        if (row_ok) epilogue_chunk(a, row, c0, r, sa_row, cs + 32 * c);
      }
      if (dead) *abort_flag = 1u;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) dq::mbar_arrive(acc_empty + acc);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPTmemCols) : "memory");
  }
}

// Any shape: one output per thread, integer dot product on CUDA cores.
__global__ void __launch_bounds__(256) w8a8_gemm_generic_kernel(const W8A8Args a) {
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t total = a.m * a.n;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = e / a.n, j = e - (e / a.n) * a.n;
    const int8_t* ar = a.a + i * a.k;
    const int8_t* br = a.b + j * a.k;
    int acc = 0;
    for (int64_t kk = 0; kk < a.k; ++kk) acc += static_cast<int>(ar[kk]) * static_cast<int>(br[kk]);
    const float scales = __fmul_rn(a.a_scale[i], a.b_scale[j]);
    store_out(a, e, __fmul_rn(__int2float_rn(acc), scales));
  }
}

// ---------------------------------------------------------------- host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// [rows, k] int8, k contiguous: 128-byte x box_rows boxes, 128-byte swizzle.
// Boxes of box_k bytes of K (128: 128-byte swizzle, 64: 64-byte swizzle) by
// box_rows rows.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t k, uint32_t box_rows, uint32_t box_k = kBK) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(k)};  // bytes between rows
  const cuuint32_t box[2] = {box_k, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, box_k == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned_to(const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) & (n - 1)) == 0; }

template <typename Kernel, typename... Args>
dq_status launch_pdl(Kernel kernel, dim3 grid, int block, size_t smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) {
    cudaGetLastError();
    return DQ_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
}

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return d;
}

constexpr dq_status kNotLaunchable = static_cast<dq_status>(-1);  // use the next path

constexpr int kMaxDevices = 64;

// Tensor-core launch of one tile configuration; kNotLaunchable when the
// tensor maps or the shared-memory opt-in are unavailable.
template <int BN, int STAGES>
dq_status launch_tc(const W8A8Args& args, int device, cudaStream_t stream) {
  using Cfg = TileConfig<BN, STAGES>;
  CUtensorMap ma, mb;
  if (!make_map(&ma, args.a, args.m, args.k, kBM) || !make_map(&mb, args.b, args.n, args.k, BN)) return kNotLaunchable;
  // the opt-in above 48 KB of dynamic shared memory, once per device
  static std::once_flag once[kMaxDevices];
  static bool ok[kMaxDevices];
  if (device < 0 || device >= kMaxDevices) return kNotLaunchable;
  std::call_once(once[device], [device] {
    ok[device] = cudaFuncSetAttribute(w8a8_gemm_tc_kernel<BN, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(Cfg::kSmemBytes)) == cudaSuccess;
    if (!ok[device]) cudaGetLastError();
  });
  if (!ok[device]) return kNotLaunchable;
  return launch_pdl(w8a8_gemm_tc_kernel<BN, STAGES>, dim3(static_cast<unsigned>((args.n + BN - 1) / BN),
                    static_cast<unsigned>((args.m + kBM - 1) / kBM)), kThreads, Cfg::kSmemBytes, stream, ma, mb, args);
}

// Persistent launch: one CTA per SM over the tile list (see
// w8a8_gemm_persistent_kernel); kNotLaunchable when the tensor maps or the
// shared-memory opt-in are unavailable.
dq_status launch_persistent(const W8A8Args& args, int device, cudaStream_t stream) {
  CUtensorMap ma, mb256, mb128;
  if (!make_map(&ma, args.a, args.m, args.k, kBM, kPBK) || !make_map(&mb256, args.b, args.n, args.k, 256, kPBK) ||
      !make_map(&mb128, args.b, args.n, args.k, 128, kPBK))
    return kNotLaunchable;
  static std::once_flag once[kMaxDevices];
  static bool ok[kMaxDevices];
  static int sms[kMaxDevices];
  if (device < 0 || device >= kMaxDevices) return kNotLaunchable;
  std::call_once(once[device], [device] {
    ok[device] = cudaFuncSetAttribute(w8a8_gemm_persistent_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(kPSmemBytes)) == cudaSuccess &&
                 cudaDeviceGetAttribute(&sms[device], cudaDevAttrMultiProcessorCount, device) == cudaSuccess &&
                 sms[device] > 0;
    if (!ok[device]) cudaGetLastError();
  });
  if (!ok[device]) return kNotLaunchable;
  const int64_t P = sms[device];
  PersistSched ps;
  ps.n_tiles = (args.n + 255) / 256;
  const int64_t T = ((args.m + kBM - 1) / kBM) * ps.n_tiles;
  const int64_t r = T % P;  // tiles of the last, partial wave
  const int64_t split = 2 * r <= P ? r : 0;  // halve them when every half gets its own SM
  ps.wide = T - split;
  ps.items = T + split;
  const int64_t grid = ps.items < P ? ps.items : P;
  return launch_pdl(w8a8_gemm_persistent_kernel, dim3(static_cast<unsigned>(grid)), kThreads, kPSmemBytes, stream,
                    ma, mb256, mb128, args, ps);
}

}  // namespace

extern "C" dq_status dq_w8a8_gemm(const int8_t* a, const int8_t* b, int64_t m, int64_t n, int64_t k,
                                  const float* a_scale, const float* b_scale, void* out, dq_dtype out_dtype,
                                  int32_t accumulate, cudaStream_t stream) {
  // k < 2^17: |sum| <= k * 128 * 128 < 2^31 for any int8 codes (-128 included)
  if (m < 0 || n < 0 || k < 1 || k >= (int64_t(1) << 17) || m > (int64_t(1) << 31) || n > (int64_t(1) << 31))
    return DQ_ERR_BAD_SHAPE;
  if (out_dtype != DQ_F32 && out_dtype != DQ_F16 && out_dtype != DQ_BF16) return DQ_ERR_BAD_DTYPE;
  if (accumulate != 0 && accumulate != 1) return DQ_ERR_BAD_ARGUMENT;
  if (accumulate && out_dtype != DQ_F32) return DQ_ERR_BAD_ARGUMENT;
  if (m == 0 || n == 0) return DQ_OK;
  if (a == nullptr || b == nullptr || a_scale == nullptr || b_scale == nullptr || out == nullptr)
    return DQ_ERR_NULL_POINTER;
  const size_t os = out_dtype == DQ_F32 ? 4 : 2;
  if (!aligned_to(a_scale, 4) || !aligned_to(b_scale, 4) || !aligned_to(out, os)) return DQ_ERR_MISALIGNED;
  // 16-byte stores need every row of out to start on a 16-byte boundary
  const bool vec = aligned_to(out, 16) && (n * static_cast<int64_t>(os)) % 16 == 0;
  W8A8Args args{a, b, a_scale, b_scale, out, m, n, k, out_dtype == DQ_F32 ? 0 : (out_dtype == DQ_F16 ? 1 : 2),
                accumulate, vec ? 1 : 0};
  // tensor maps need 16-byte row pitches (k % 16 == 0) and bases; ragged m,
  // n and k are zero-filled by the loads and masked in the epilogue
  const bool tiles = k % 16 == 0 && (m + kBM - 1) / kBM <= 65535 && aligned_to(a, 16) && aligned_to(b, 16);
  if (tiles) {
    const int device = current_device();
#ifndef DQ_W8A8_NO_PERSISTENT
    const dq_status pst = launch_persistent(args, device, stream);
    if (pst != kNotLaunchable) return pst;
#endif
    // 256-wide tiles unless a 128-wide last tile would waste less
    if (DQ_W8A8_BN >= 256 && (n % 256 == 0 || n % 256 > 128)) {
      const dq_status st = launch_tc<256, DQ_W8A8_STAGES_256>(args, device, stream);
      if (st != kNotLaunchable) return st;
    }
    const dq_status st = launch_tc<128, DQ_W8A8_STAGES_128>(args, device, stream);
    if (st != kNotLaunchable) return st;
  }
  const int64_t total = m * n;
  int64_t grid = (total + 255) / 256;
  if (grid > 148 * 64) grid = 148 * 64;
  return launch_pdl(w8a8_gemm_generic_kernel, dim3(static_cast<unsigned>(grid)), 256, 0, stream, args);
}
