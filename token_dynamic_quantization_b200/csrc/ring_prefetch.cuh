// L2 prefetch of a ring kernel's first rows, issued before the kernel's
// griddepcontrol.wait so that the row copies after the wait find their bytes
// in L2 instead of waiting for HBM (sm_100a).
#pragma once

#include <stdint.h>

namespace dq {

// L2 prefetch of `bytes` (multiple of 16) at a 16-byte aligned global
// address: a hint that returns no data to the thread. L2 is the device's
// point of coherence, so a copy issued after griddepcontrol.wait still reads
// what the kernel before wrote, even where the prefetch ran before the wait.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src_gmem, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src_gmem), "r"(bytes) : "memory");
}

// Rows of the CTA's range a ring kernel prefetches into L2 before its
// griddepcontrol.wait: about DQ_RING_PREFETCH_BYTES, at least one row, at
// most the ring and the range. Measured per call over 20 calls (8192 x 4096
// bf16 with smooth scales / 4 x 4096 x 3072 AdaLayerNorm): none 18.3 / 35.1
// us, 24 KB 17.8 / 34.5, 48 KB 17.4 / 34.0, 72 KB 17.5 / 34.3, the whole
// ring (96 KB) 17.9 / 34.3, twice the ring 18.7 / 36.0. More prefetched
// bytes delay the first copies after the wait.
#ifndef DQ_RING_PREFETCH_BYTES
#define DQ_RING_PREFETCH_BYTES 49152u
#endif
__device__ __forceinline__ int ring_prefetch_rows(uint32_t row_bytes, int slots, int n) {
  int rows = static_cast<int>(DQ_RING_PREFETCH_BYTES / row_bytes);
  rows = rows < 1 ? 1 : (rows > slots ? slots : rows);
  return rows < n ? rows : n;
}

}  // namespace dq
