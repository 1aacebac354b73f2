// The two Ulysses all-to-alls, held inside one GPU's HBM as layout
// permutations ("Paralelismul de Secvență Ulysses", section "Mecanismul de
// funcționare Ulysses", steps 3 and 5):
//
//   seq layout  X[r][b][tt][hg][:]   (rank r holds positions t = r*s + tt)
//   head layout X[r2][b][hh][t][:]   (rank r2 holds heads hg = r2*hl + hh)
//
// Both directions move whole rows of head_dim elements, so they are byte
// copies, bit-exact for any element type.
//
// Main path, staged through TMA: a persistent CTA per SM, one thread, moves
// blocks of TOK consecutive positions of one (rank, batch) pair.  The seq-side
// tensor map is declared with its position dimension before its head
// dimension, so ONE tensor load brings the block's TOK x heads rows into
// shared memory in [head][position] order, and each destination rank r2's
// hl heads leave with one store through a head-side map (head->seq: the
// reverse, P loads and one store).  The transpose is done by the maps' strides:
// no per-element index arithmetic, every row moved as a whole (rows >= 16 B).
// Blocks stream through a ring of three 64 KB stages, loads running ahead of
// stores.  Several tensors (Q, K, V) can share one launch.
//
// Fallback for shapes the maps cannot express (more than 256 heads, rows over
// 1 KB, a stage over 64 KB): a vector kernel in which a CTA owns a run of TOK
// consecutive tokens of one (rank, batch) pair and copies 16-byte vectors,
// coalesced on both sides.
#include "common.cuh"
#include "prof.cuh"
#include "sm100.cuh"

namespace uly {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 8;  // 16-byte vectors in flight per thread

// VPR = 16-byte vectors per row (row_bytes / 16).  TO_HEAD selects direction.
template <int VPR, bool TO_HEAD>
__global__ void __launch_bounds__(kThreads) permute_rows_kernel(
    const uint4 *__restrict__ src, uint4 *__restrict__ dst, int B, int n, int s, int heads,
    int hl, int tok_per_cta) {
  const int rb = blockIdx.y;        // r * B + b
  const int r = rb / B, b = rb - r * B;
  const int tt0 = blockIdx.x * tok_per_cta;
  const int ntok = min(tok_per_cta, s - tt0);
  if (ntok <= 0) return;
  const long long total = (long long)ntok * heads * VPR;  // vectors of this CTA
  // seq side: the CTA's block starts at row ((r*B + b)*s + tt0)*heads
  const long long seq_row0 = ((long long)rb * s + tt0) * heads;

  for (long long base = (long long)threadIdx.x; base < total; base += (long long)kThreads * kUnroll) {
    uint4 v[kUnroll];
    long long head_vec[kUnroll];
    long long seq_vec[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long e = base + (long long)u * kThreads;  // vector index in the CTA block
      if (e < total) {
        const int row = (int)(e / VPR), lane = (int)(e % VPR);
        const int tok = row / heads, hg = row - tok * heads;
        const int r2 = hg / hl, hh = hg - r2 * hl;
        const long long t = (long long)r * s + tt0 + tok;
        seq_vec[u] = (seq_row0 + row) * VPR + lane;
        head_vec[u] = ((((long long)r2 * B + b) * hl + hh) * n + t) * VPR + lane;
        v[u] = TO_HEAD ? __ldcs(src + seq_vec[u]) : __ldcs(src + head_vec[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long e = base + (long long)u * kThreads;
      if (e < total) {
        if (TO_HEAD) __stcs(dst + head_vec[u], v[u]);
        else __stcs(dst + seq_vec[u], v[u]);
      }
    }
  }
}

template <bool TO_HEAD>
cudaError_t launch_permute(int B, int n, int P, int heads, int vpr, const void *src, void *dst,
                           cudaStream_t stream) {
  const int s = n / P, hl = heads / P;
  // about 4096 vectors (64 KB) per CTA
  int tok = 4096 / (heads * vpr);
  if (tok < 1) tok = 1;
  if (tok > s) tok = s;
  dim3 grid((s + tok - 1) / tok, P * B);
  const uint4 *in = static_cast<const uint4 *>(src);
  uint4 *out = static_cast<uint4 *>(dst);
  prof::Scope scope(TO_HEAD ? prof::K_SEQ_TO_HEAD_VEC : prof::K_HEAD_TO_SEQ_VEC, stream);
#define ULY_PERMUTE_CASE(V)                                                                   \
  case V:                                                                                     \
    permute_rows_kernel<V, TO_HEAD><<<grid, kThreads, 0, stream>>>(in, out, B, n, s, heads, \
                                                                   hl, tok);                  \
    break;
  switch (vpr) {
    ULY_PERMUTE_CASE(1)
    ULY_PERMUTE_CASE(2)
    ULY_PERMUTE_CASE(4)
    ULY_PERMUTE_CASE(8)
    ULY_PERMUTE_CASE(16)
    ULY_PERMUTE_CASE(32)
    ULY_PERMUTE_CASE(64)
    default:
      return cudaErrorInvalidValue;
  }
#undef ULY_PERMUTE_CASE
  note_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------ TMA path
constexpr int kMaxItems = 4;
constexpr int kTmaStages = 3;
constexpr uint32_t kTmaStageBytes = 65536;
constexpr uint32_t kTmaSmem = kTmaStages * kTmaStageBytes + 1024 + 64;   // stages, alignment, barriers

struct TmaItem {
  int tok;                  // positions per block (power of two, 8..256)
  int tok_blocks;           // ceil(s / tok)
  long long block_begin;    // first block of this tensor in the launch
  uint32_t stage_bytes;     // heads * tok * row bytes
  uint32_t rank_bytes;      // hl * tok * row bytes: one destination rank's heads
};
struct TmaBatch {
  TmaItem it[kMaxItems];
  int count, B, P;
  long long total_blocks;
  int *err;
};
// seq[i]: dims (row words, s, heads, P*B) -- the position dimension before the
// head dimension, so a box lands as [head][position][row];
// head[i]: dims (row words, s, P, hl, P*B) over [r2][b][hl][n = P*s][row].
struct TmaMaps {
  CUtensorMap seq[kMaxItems];
  CUtensorMap head[kMaxItems];
};

template <bool TO_HEAD>
__global__ void __launch_bounds__(32, 1) permute_tma_kernel(const __grid_constant__ TmaMaps maps,
                                                             const TmaBatch bt) {
  using namespace sm100;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  if (threadIdx.x != 0) return;
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kTmaStages * kTmaStageBytes);
  for (int i = 0; i < kTmaStages; ++i) mbar_init(smem_u32(&bars[i]), 1);
  fence_mbar_init();
  for (int i = 0; i < bt.count; ++i) {
    tma_prefetch_desc(&maps.seq[i]);
    tma_prefetch_desc(&maps.head[i]);
  }
  const long long nlocal =
      bt.total_blocks > blockIdx.x ? (bt.total_blocks - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  // block k of this CTA: tensor i, (rank r, batch b) = rb, positions [tt0, tt0 + tok)
  auto decode = [&](long long k, int &i, int &rb, int &tt0) {
    const long long g = blockIdx.x + k * gridDim.x;
    i = 0;
    while (i + 1 < bt.count && g >= bt.it[i + 1].block_begin) ++i;
    const long long local = g - bt.it[i].block_begin;
    rb = (int)(local / bt.it[i].tok_blocks);
    tt0 = (int)(local - (long long)rb * bt.it[i].tok_blocks) * bt.it[i].tok;
  };
  auto issue_load = [&](long long k) {
    int i, rb, tt0;
    decode(k, i, rb, tt0);
    const int st = (int)(k % kTmaStages);
    const uint32_t dst = sb + st * kTmaStageBytes, bar = smem_u32(&bars[st]);
    mbar_arrive_expect_tx(bar, bt.it[i].stage_bytes);
    if (TO_HEAD) {
      tma_load_4d(dst, &maps.seq[i], bar, 0, tt0, 0, rb);
    } else {
      const int r = rb / bt.B, b = rb - r * bt.B;
      for (int r2 = 0; r2 < bt.P; ++r2)
        tma_load_5d(dst + r2 * bt.it[i].rank_bytes, &maps.head[i], bar, 0, tt0, r, 0, r2 * bt.B + b);
    }
  };
  auto issue_store = [&](long long k) {
    int i, rb, tt0;
    decode(k, i, rb, tt0);
    const uint32_t src = sb + (int)(k % kTmaStages) * kTmaStageBytes;
    if (TO_HEAD) {
      const int r = rb / bt.B, b = rb - r * bt.B;
      for (int r2 = 0; r2 < bt.P; ++r2)
        tma_store_5d(&maps.head[i], src + r2 * bt.it[i].rank_bytes, 0, tt0, r, 0, r2 * bt.B + b);
    } else {
      tma_store_4d(&maps.seq[i], src, 0, tt0, 0, rb);
    }
    bulk_commit_group();
  };
  long long issued = 0;
  for (; issued < nlocal && issued < kTmaStages; ++issued) issue_load(issued);
  long long k = 0;
  for (; k < nlocal; ++k) {
    const int st = (int)(k % kTmaStages);
    if (!mbar_wait(smem_u32(&bars[st]), (uint32_t)((k / kTmaStages) & 1), nullptr, bt.err)) break;
    issue_store(k);
    // refill the previous block's stage once its stores have read it
    if (k >= 1 && issued < nlocal) {
      bulk_wait_group_read<1>();
      issue_load(issued++);
    }
  }
  // every load issued lands (also after a wait that ran out), every store completes
  for (; k < issued; ++k)
    mbar_wait(smem_u32(&bars[k % kTmaStages]), (uint32_t)((k / kTmaStages) & 1), nullptr, bt.err);
  bulk_wait_all();
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// The two maps of one tensor (see TmaMaps) and its block geometry; false when
// the shape is outside what the TMA path handles.
bool tma_item(const void *seq_base, const void *head_base, int B, int n, int P, int heads, int row_bytes,
              CUtensorMap *mseq, CUtensorMap *mhead, TmaItem *it) {
  const int s = n / P, hl = heads / P, words = row_bytes / 4;
  if (heads > 256 || words > 256 || row_bytes % 16) return false;
  int tok = 8;
  while (tok < 256 && (uint64_t)heads * row_bytes * (tok * 2) <= kTmaStageBytes && tok < s) tok *= 2;
  if ((uint64_t)heads * row_bytes * tok > kTmaStageBytes) return false;
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t rb = (cuuint64_t)row_bytes;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  {
    cuuint64_t dims[4] = {(cuuint64_t)words, (cuuint64_t)s, (cuuint64_t)heads, (cuuint64_t)P * B};
    cuuint64_t strides[3] = {rb * heads, rb, rb * heads * s};
    cuuint32_t box[4] = {(cuuint32_t)words, (cuuint32_t)tok, (cuuint32_t)heads, 1};
    if (enc(mseq, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<void *>(seq_base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  {
    cuuint64_t dims[5] = {(cuuint64_t)words, (cuuint64_t)s, (cuuint64_t)P, (cuuint64_t)hl, (cuuint64_t)P * B};
    cuuint64_t strides[4] = {rb, rb * s, rb * n, rb * n * hl};
    cuuint32_t box[5] = {(cuuint32_t)words, (cuuint32_t)tok, 1, (cuuint32_t)hl, 1};
    if (enc(mhead, CU_TENSOR_MAP_DATA_TYPE_UINT32, 5, const_cast<void *>(head_base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  it->tok = tok;
  it->tok_blocks = (s + tok - 1) / tok;
  it->stage_bytes = (uint32_t)((uint64_t)heads * row_bytes * tok);
  it->rank_bytes = (uint32_t)((uint64_t)hl * row_bytes * tok);
  return true;
}

}  // namespace

// Up to kMaxItems tensors of the same (B, n, P, row) in one launch; false when
// the TMA path does not cover the shapes (the caller then uses the vector kernel).
bool permute_tma_try(bool to_head, int B, int n, int P, int row_bytes, int count, const void *const *srcs,
                     void *const *dsts, const int *heads, cudaStream_t stream, uly_status *st) {
  if (count < 1 || count > kMaxItems) return false;
  TmaMaps maps;
  TmaBatch bt;
  bt.count = count;
  bt.B = B;
  bt.P = P;
  long long total = 0;
  for (int i = 0; i < count; ++i) {
    const void *seq_base = to_head ? srcs[i] : dsts[i];
    const void *head_base = to_head ? dsts[i] : srcs[i];
    if (!tma_item(seq_base, head_base, B, n, P, heads[i], row_bytes, &maps.seq[i], &maps.head[i], &bt.it[i]))
      return false;
    bt.it[i].block_begin = total;
    total += (long long)bt.it[i].tok_blocks * P * B;
  }
  for (int i = count; i < kMaxItems; ++i) {
    maps.seq[i] = maps.seq[0];
    maps.head[i] = maps.head[0];
    bt.it[i] = bt.it[0];
    bt.it[i].block_begin = total;
  }
  bt.total_blocks = total;
  bt.err = error_word();
  static std::atomic<uint64_t> optin_to_head{0}, optin_to_seq{0};
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    *st = ULY_ERR_CUDA;
    return true;
  }
  const bool opted = to_head ? smem_optin(permute_tma_kernel<true>, kTmaSmem, optin_to_head)
                             : smem_optin(permute_tma_kernel<false>, kTmaSmem, optin_to_seq);
  if (!opted) {
    *st = ULY_ERR_CUDA;
    return true;
  }
  const int grid = (int)(total < sms ? total : sms);
  if (grid > 0) {
    prof::Scope scope(to_head ? prof::K_SEQ_TO_HEAD : prof::K_HEAD_TO_SEQ, stream);
    if (to_head)
      permute_tma_kernel<true><<<grid, 32, kTmaSmem, stream>>>(maps, bt);
    else
      permute_tma_kernel<false><<<grid, 32, kTmaSmem, stream>>>(maps, bt);
    note_launches(1);
  }
  *st = last_launch_status();
  return true;
}

uly_status permute_validate(int32_t B, int32_t n, int32_t P, int32_t heads, int32_t d,
                            int32_t elem_bytes, const void *src, const void *dst) {
  if (!src || !dst) return ULY_ERR_NULL;
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8) return ULY_ERR_DTYPE;
  if (B <= 0 || n <= 0 || P <= 0 || heads <= 0 || d <= 0) return ULY_ERR_SHAPE;
  if (n % P || heads % P) return ULY_ERR_SHAPE;
  if (B > 65535 / P) return ULY_ERR_SHAPE;  // grid.y = P * B
  const long long row = (long long)d * elem_bytes;
  if (row % 16) return ULY_ERR_ALIGN;
  const long long vpr = row / 16;
  if (vpr > 64 || (vpr & (vpr - 1))) return ULY_ERR_UNSUPPORTED;
  if (!aligned16(src) || !aligned16(dst)) return ULY_ERR_ALIGN;
  const size_t bytes = (size_t)B * n * heads * row;
  if (overlap(src, bytes, dst, bytes)) return ULY_ERR_ALIAS;
  return ULY_OK;
}

// Several tensors of the same (B, n, P, d, element size): one TMA launch when
// it covers them, else one vector-kernel launch per tensor.
uly_status permute_batch_launch(bool to_head, int32_t B, int32_t n, int32_t P, int32_t d, int32_t elem_bytes,
                                int32_t count, const uly_permute_item *items, cudaStream_t stream) {
  const void *srcs[kMaxItems];
  void *dsts[kMaxItems];
  int heads[kMaxItems];
  for (int i = 0; i < count; ++i) {
    srcs[i] = items[i].src;
    dsts[i] = items[i].dst;
    heads[i] = items[i].heads;
  }
  uly_status st = ULY_OK;
  if (permute_tma_try(to_head, B, n, P, d * elem_bytes, count, srcs, dsts, heads, stream, &st)) return st;
  const int vpr = (int)((long long)d * elem_bytes / 16);
  for (int i = 0; i < count; ++i) {
    cudaError_t e = to_head ? launch_permute<true>(B, n, P, heads[i], vpr, srcs[i], dsts[i], stream)
                            : launch_permute<false>(B, n, P, heads[i], vpr, srcs[i], dsts[i], stream);
    if (e != cudaSuccess) return ULY_ERR_CUDA;
  }
  return ULY_OK;
}

uly_status permute_launch(bool to_head, int32_t B, int32_t n, int32_t P, int32_t heads, int32_t d,
                          int32_t elem_bytes, const void *src, void *dst, cudaStream_t stream) {
  uly_status st = ULY_OK;
  void *dsts[1] = {dst};
  if (permute_tma_try(to_head, B, n, P, d * elem_bytes, 1, &src, dsts, &heads, stream, &st)) return st;
  const int vpr = (int)((long long)d * elem_bytes / 16);
  cudaError_t e = to_head ? launch_permute<true>(B, n, P, heads, vpr, src, dst, stream)
                          : launch_permute<false>(B, n, P, heads, vpr, src, dst, stream);
  return e == cudaSuccess ? ULY_OK : ULY_ERR_CUDA;
}

}  // namespace uly
