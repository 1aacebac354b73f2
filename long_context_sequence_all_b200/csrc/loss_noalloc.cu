// ulysses_loss_aggregate_noalloc: the token-weighted loss aggregation for
// callers that cannot allocate device memory.
//
// Some callers only ever hand the library the buffers of their inputs and
// outputs: plugin hosts and runtimes that own every device allocation
// themselves, or processes that forbid device allocation after start-up to
// keep a fixed memory budget.  They cannot obtain the few KB of workspace
// ulysses_loss_aggregate needs for its per-CTA partial sums.  This entry point
// runs the same two kernels with that scratch taken from a fixed array that
// is part of the library image instead.
//
// Costs and rules of that array:
//  - It is kNoAllocScratchBytes (64 KiB) of device memory on every GPU that
//    loads the library, held until the process exits.
//  - Shapes whose partials do not fit (more than 4096 partial sums, i.e.
//    P * blocks-per-shard > 4096; about P > 3500 ranks) are rejected with
//    ULY_ERR_WORKSPACE before anything is launched.
//  - Every call uses the same array and it keeps the last call's contents.
//    Nothing in it has to start at zero: each partial slot is written by one
//    CTA of the first kernel before the second kernel of the same call reads
//    it.  Calls that overlap on the GPU (different streams, no ordering
//    between them) race on the array and give wrong results.
//  - The first call on a device looks up the array's device address on that
//    device (cudaGetSymbolAddress), so that first call should come before any
//    stream capture.
// No cudaMalloc, cudaFree or other allocating routine is called.
#include <mutex>

#include "common.cuh"

namespace uly {

size_t loss_workspace_bytes(int P, long long per_shard);
uly_status loss_validate(int32_t, int64_t, int32_t, int32_t, const void *, const int32_t *,
                         const float *, const int64_t *, const float *);
uly_status loss_launch(int32_t, int64_t, int32_t, int32_t, const void *, const int32_t *, int32_t,
                       float *, int64_t *, float *, void *, cudaStream_t);

namespace {

constexpr size_t kNoAllocScratchBytes = ULYSSES_NOALLOC_LOSS_SCRATCH_BYTES;

// The scratch itself.  In host code this name is only a host-side handle of
// the symbol, not a device address: kernels receive the address looked up
// below.
static __device__ __align__(256) unsigned char g_loss_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void *g_scratch[64] = {nullptr};

// Device address of the scratch on the current device (looked up once per
// device, with that device current); nullptr if the lookup fails.
void *scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_loss_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch[dev] = p;
  }
  return g_scratch[dev];
}

}  // namespace
}  // namespace uly

using namespace uly;

extern "C" uly_status ulysses_loss_aggregate_noalloc(int32_t world, int64_t tokens, int32_t vocab,
                                                     int32_t logit_dtype, const void *logits,
                                                     const int32_t *labels, int32_t ignore_index,
                                                     float *shard_sum, int64_t *shard_count,
                                                     float *loss, void *stream) {
  uly_status st = loss_validate(world, tokens, vocab, logit_dtype, logits, labels, shard_sum,
                                shard_count, loss);
  if (st != ULY_OK) return st;
  if (loss_workspace_bytes(world, tokens / world) > kNoAllocScratchBytes) return ULY_ERR_WORKSPACE;
  const size_t zb = (size_t)tokens * vocab * (logit_dtype == ULY_BF16 ? 2 : 4);
  const size_t yb = (size_t)tokens * 4;
  const void *outs[3] = {shard_sum, shard_count, loss};
  const size_t outb[3] = {(size_t)world * 4, (size_t)world * 8, 4};
  for (int a = 0; a < 3; ++a)
    if (overlap(outs[a], outb[a], logits, zb) || overlap(outs[a], outb[a], labels, yb))
      return ULY_ERR_ALIAS;
  void *scratch = scratch_address();
  if (!scratch) return ULY_ERR_CUDA;
  return loss_launch(world, tokens, vocab, logit_dtype, logits, labels, ignore_index, shard_sum,
                     shard_count, loss, scratch, static_cast<cudaStream_t>(stream));
}
