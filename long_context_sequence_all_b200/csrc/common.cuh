// Internal helpers shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>

#include "ulysses.h"

namespace uly {

// Data-dependent failures are OR-ed as (1 << status) into the device error
// word of the current device (see error_word()); kernels never trap.
// err[0] is the word; err[1..kErrInfoWords) describe the first bounded wait
// that ran out (see ulysses_read_error_info).
constexpr int kErrInfoWords = 16;
__device__ __forceinline__ void raise_error(int *err, uly_status s) {
  if (err) atomicOr(err, 1 << (int)s);
}

// Device address of the error record of the current device (nullptr on failure).
int *error_word();

// Host-side launch bookkeeping (counts every kernel launched by the library).
void note_launches(int n);

// Cycles a pipeline wait of the tcgen05 kernels may last before it reports
// ULY_ERR_TIMEOUT: the built-in limit, or a shorter one a test set with
// ulysses_set_wait_limit (read by the launchers into the kernel parameters).
long long wait_limit_cycles();
// The attention kernels' block order set with ulysses_set_attn_block_order
// (ULY_BLOCK_ORDER_*; read by the launchers).
int attn_block_order();

inline uly_status last_launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ULY_OK : ULY_ERR_CUDA;
}

// Opt `kernel` into `bytes` of dynamic shared memory on the current device.
// The attribute belongs to a device, so it is set once per device; `done`
// holds one bit per device already set (atomic: host threads may race here).
template <typename Kernel>
inline bool smem_optin(Kernel kernel, int bytes, std::atomic<uint64_t> &done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  const uint64_t bit = uint64_t(1) << dev;
  if (done.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  done.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Streaming multiprocessors of the current device (148, a B200's count, if
// the query fails).
inline int device_sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return 148;
  return sms;
}

// Block order of the attention kernels.  Starting the CTAs of one KV head at
// a time keeps the K/V (forward) or Q/dO and dQ rows (backward) of one GQA
// group in L2; starting the heaviest tiles of every head first balances the
// SMs' load best.  Under a causal mask the heaviest CTA does twice the
// average, so taking the heads one at a time leaves no tail only when a
// head's CTAs along the sequence are more than twice the SMs (64K tokens on
// a B200: yes; 8K: no).  Document masks bound each CTA's work by its
// document and gain little from the locality; they keep the balanced order.
// ulysses_set_attn_block_order can fix either order (for tests that compare
// them); the results do not depend on it (dQ of the fused backward aside,
// whose fp32 adds meet in L2 in run-dependent order either way).
inline bool attn_kv_head_major(int mask, long long ctas_per_kv_head) {
  const int order = attn_block_order();
  if (order == ULY_BLOCK_ORDER_KV_HEAD_MAJOR) return true;
  if (order == ULY_BLOCK_ORDER_HEAVIEST_FIRST) return false;
  return mask != ULY_MASK_DOC_CAUSAL && ctas_per_kv_head > 2LL * device_sm_count();
}

inline bool overlap(const void *a, size_t na, const void *b, size_t nb) {
  uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Position ranges of the three masks.  Row i may see keys [lo, hi].
// doc-causal: the document containing i, found by binary search in cu_seqlens.
// A well-formed cu_seqlens (cu[0] = 0, non-decreasing, cu[num_docs] = n) is
// checked on the device by check_cu_seqlens_kernel; the bounds returned here
// are clamped to [0, i] and [i + 1, n] so that a malformed one can only give a
// wrong mask, never a tile outside the operands.
__device__ __forceinline__ int doc_index_of(const int32_t *__restrict__ cu, int num_docs, int i) {
  int lo = 0, hi = num_docs - 1;  // find the largest e with cu[e] <= i
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}
__device__ __forceinline__ int doc_start_of(const int32_t *__restrict__ cu, int num_docs, int i) {
  return min(max(__ldg(cu + doc_index_of(cu, num_docs, i)), 0), i);
}
__device__ __forceinline__ int doc_end_of(const int32_t *__restrict__ cu, int num_docs, int i, int n) {
  return min(max(__ldg(cu + doc_index_of(cu, num_docs, i) + 1), i + 1), n);
}

struct MaskInfo {
  int mask;            // uly_mask
  int n;
  const int32_t *cu;
  int num_docs;
  // visible keys of query row i (i < n): [lo, hi]
  __device__ __forceinline__ void row_range(int i, int &lo, int &hi) const {
    if (mask == ULY_MASK_NONE) { lo = 0; hi = n - 1; return; }
    hi = i;
    lo = (mask == ULY_MASK_DOC_CAUSAL) ? doc_start_of(cu, num_docs, i) : 0;
  }
  // query rows that see key j (j < n): [lo, hi]
  __device__ __forceinline__ void col_range(int j, int &lo, int &hi) const {
    if (mask == ULY_MASK_NONE) { lo = 0; hi = n - 1; return; }
    lo = j;
    hi = (mask == ULY_MASK_DOC_CAUSAL) ? doc_end_of(cu, num_docs, j, n) - 1 : n - 1;
  }
};

// Workspace of the bf16 backward: D_i and LSE_i log2(e) per query row, each
// head's rows padded to a multiple of 128 so every 128-row tile of them is one
// aligned 512-byte block; the LSE array starts bwd_stats_stride floats after D.
__host__ __device__ inline int bwd_rows_padded(int n) { return (n + 127) / 128 * 128; }
__host__ __device__ inline long long bwd_stats_stride(long long rows_pad) { return (rows_pad + 63) / 64 * 64; }

// Row of the seq layout [P][B][n/P][heads][d] that holds row t of head hx of
// the head layout [P][B][hl][n][d] (hx = (r*B + b)*hl + hh, heads = P*hl):
// rank t / (n/P), position t % (n/P), global head r*hl + hh.  This is the
// second all-to-all (step 5) for one row.
__host__ __device__ inline long long seq_row_of(long long hx, int t, int B, int n, int P, int hl) {
  const int s = n / P;
  const long long bh = (long long)B * hl;
  const long long r = hx / bh;
  const long long rem = hx - r * bh;
  const long long b = rem / hl, hh = rem - b * hl;
  const int rt = t / s, tt = t - rt * s;
  return (((long long)rt * B + b) * s + tt) * ((long long)P * hl) + r * hl + hh;
}

// Per-launch geometry of the head layout shared by the attention kernels.
struct HeadGeom {
  int B, n, P, hl, gl, group;  // hl = H/P, gl = G/P, group = H/G
  float scale;                 // softmax scale
  int out_seq;                 // 1: outputs go to the seq layout (uly_attn_desc.out_seq_layout)
  // output row of query-head row (qh, t) and of KV-head row (kvh, t)
  __host__ __device__ long long q_out_row(long long qh, int t) const {
    return out_seq ? seq_row_of(qh, t, B, n, P, hl) : qh * n + t;
  }
  __host__ __device__ long long kv_out_row(long long kvh, int t) const {
    return out_seq ? seq_row_of(kvh, t, B, n, P, gl) : kvh * n + t;
  }
};

}  // namespace uly
