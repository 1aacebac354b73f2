// Label shift before sharding (next-token labels over the whole sequence).
#include "common.cuh"
#include "prof.cuh"

namespace uly {

// Next-token labels, shifted on the whole sequence before it is sharded: the
// last position of shard r is labelled with the first token of shard r+1
// (the SFT trainer's automatic label shift: "Ulysses 序列平行化", section
// "在 Hugging Face 生態系統中的整合"; padding to a multiple of sp_size and
// packed variable-length sequences: "Paralelismul de Secvență Ulysses",
// section "Integrarea cu Transformers Trainer și TRL SFTTrainer").
//   label(t) = ids[t+1]       if t+1 < valid_len and t+1 starts no document
//            = ignore_index   otherwise
// One thread per output label, written in seq layout [P][B][n/P]; reads of
// ids are coalesced along each (rank, batch) run.  Document starts come from
// a binary search of the sorted cu_seqlens (the same array attention uses).
namespace {
__global__ void shift_labels_kernel(const int32_t *__restrict__ ids, const int32_t *__restrict__ cu,
                                    int num_docs, int B, int n, int s, int valid_len,
                                    int ignore_index, int32_t *__restrict__ labels) {
  const long long total = (long long)B * n;
  for (long long o = (long long)blockIdx.x * blockDim.x + threadIdx.x; o < total;
       o += (long long)gridDim.x * blockDim.x) {
    const long long rb = o / s;
    const int tt = (int)(o - rb * s);
    const int r = (int)(rb / B), b = (int)(rb - (long long)r * B);
    const int t = r * s + tt;
    int y = ignore_index;
    if (t + 1 < valid_len) {
      const bool starts = cu != nullptr && doc_start_of(cu, num_docs, t + 1) == t + 1;
      if (!starts) y = __ldg(ids + (long long)b * n + t + 1);
    }
    labels[o] = y;
  }
}
}  // namespace

uly_status shift_labels_launch(int32_t B, int32_t n, int32_t P, const int32_t *ids,
                               const int32_t *cu, int32_t num_docs, int32_t valid_len,
                               int32_t ignore_index, int32_t *labels, cudaStream_t stream) {
  const long long total = (long long)B * n;
  long long blocks = (total + 255) / 256;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  prof::Scope scope(prof::K_SHIFT_LABELS, stream);
  shift_labels_kernel<<<(unsigned)blocks, 256, 0, stream>>>(ids, num_docs > 0 ? cu : nullptr,
                                                            num_docs, B, n, n / P, valid_len,
                                                            ignore_index, labels);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? ULY_OK : ULY_ERR_CUDA;
}

}  // namespace uly
