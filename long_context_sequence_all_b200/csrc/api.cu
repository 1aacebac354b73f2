// C ABI of the Ulysses attention layer: argument validation and dispatch to
// the kernels.  Declarations and the contract of every entry point are in
// include/ulysses.h.  Nothing here allocates device memory.
#include <atomic>
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "prof.cuh"

namespace uly {

// Device error word, one per device context (module globals are per context).
__device__ int g_error_word_storage[kErrInfoWords] = {0};

namespace {
std::atomic<uint64_t> g_launches{0};
std::mutex g_err_mu;
int *g_err_ptr[64] = {nullptr};
}  // namespace

void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

namespace {
constexpr long long kDefaultWaitLimit = 2000000000ll;   // sm100::kWaitLimitCycles
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};
}  // namespace

long long wait_limit_cycles() { return g_wait_limit.load(std::memory_order_relaxed); }

namespace {
std::atomic<int> g_attn_block_order{ULY_BLOCK_ORDER_AUTO};
}  // namespace

int attn_block_order() { return g_attn_block_order.load(std::memory_order_relaxed); }

int *error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word_storage) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<int *>(p);
  }
  return g_err_ptr[dev];
}

// launchers implemented in the kernel translation units
uly_status permute_validate(int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, const void *,
                            const void *);
uly_status permute_launch(bool, int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, const void *,
                          void *, cudaStream_t);
uly_status permute_batch_launch(bool, int32_t, int32_t, int32_t, int32_t, int32_t, int32_t,
                                const uly_permute_item *, cudaStream_t);
uly_status attn_f32_fwd_launch(const uly_attn_desc *, const HeadGeom &, const MaskInfo &,
                               const void *, const void *, const void *, void *, float *,
                               cudaStream_t);
uly_status attn_f32_bwd_launch(const uly_attn_desc *, const HeadGeom &, const MaskInfo &,
                               const void *, const void *, const void *, const void *,
                               const float *, const void *, void *, void *, void *, float *,
                               cudaStream_t);
uly_status attn_bf16_fwd_launch(const uly_attn_desc *, const HeadGeom &, const MaskInfo &,
                                const void *, const void *, const void *, void *, float *,
                                cudaStream_t);
size_t attn_bf16_bwd_workspace(const HeadGeom &, bool);
uly_status attn_bf16_bwd_launch(const uly_attn_desc *, const HeadGeom &, const MaskInfo &,
                                const void *, const void *, const void *, const void *,
                                const float *, const void *, void *, void *, void *, float *,
                                cudaStream_t);
uly_status kv_rep_validate(int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, const void *,
                           const void *);
uly_status kv_replicate_launch(int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, const void *,
                               void *, cudaStream_t);
uly_status kv_reduce_launch(int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, const void *, void *,
                            cudaStream_t);
uly_status shift_labels_launch(int32_t, int32_t, int32_t, const int32_t *, const int32_t *, int32_t,
                               int32_t, int32_t, int32_t *, cudaStream_t);
uly_status rope_table_launch(int32_t, int32_t, double, float *, cudaStream_t);
uly_status qkv_proj_launch(int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, const void *, const void *,
                           const float *, int32_t, const int32_t *, void *, void *, void *, cudaStream_t);
uly_status o_proj_launch(int32_t, int32_t, int32_t, int32_t, int32_t, const void *, const void *, void *,
                         cudaStream_t);
uly_status qkv_proj_bwd_launch(int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, const void *, const void *,
                               const float *, int32_t, const int32_t *, const void *, const void *, const void *,
                               void *, float *, void *, cudaStream_t);
uly_status o_proj_bwd_launch(int32_t, int32_t, int32_t, int32_t, int32_t, const void *, const void *, const void *,
                             void *, float *, cudaStream_t);
size_t loss_workspace_bytes(int P, long long per_shard);
size_t loss_bwd_workspace_bytes(int P, long long per_shard);
uly_status loss_bwd_launch(int32_t, int64_t, int32_t, int32_t, const void *, const int32_t *, int32_t,
                           void *, float *, int64_t *, float *, void *, cudaStream_t);
uly_status loss_validate(int32_t, int64_t, int32_t, int32_t, const void *, const int32_t *,
                         const float *, const int64_t *, const float *);
uly_status loss_launch(int32_t, int64_t, int32_t, int32_t, const void *, const int32_t *, int32_t,
                       float *, int64_t *, float *, void *, cudaStream_t);

namespace {

uly_status check_desc(const uly_attn_desc *d, HeadGeom &g, MaskInfo &mk) {
  if (!d) return ULY_ERR_NULL;
  if (d->batch <= 0 || d->seq_len <= 0 || d->world <= 0 || d->n_q_heads <= 0 || d->n_kv_heads <= 0 ||
      d->head_dim <= 0)
    return ULY_ERR_SHAPE;
  if (d->seq_len % d->world || d->n_q_heads % d->world || d->n_kv_heads % d->world ||
      d->n_q_heads % d->n_kv_heads)
    return ULY_ERR_SHAPE;
  if (d->dtype != ULY_F32 && d->dtype != ULY_BF16) return ULY_ERR_DTYPE;
  if (d->mask < ULY_MASK_NONE || d->mask > ULY_MASK_DOC_CAUSAL) return ULY_ERR_UNSUPPORTED;
  if (d->mask == ULY_MASK_DOC_CAUSAL && (!d->cu_seqlens || d->num_docs < 1)) return ULY_ERR_NULL;
  if (!(d->softmax_scale >= 0.f) || !std::isfinite(d->softmax_scale)) return ULY_ERR_SHAPE;
  if ((d->out_seq_layout != 0 && d->out_seq_layout != 1) || (d->deterministic != 0 && d->deterministic != 1))
    return ULY_ERR_SHAPE;
  const long long heads_q = (long long)d->batch * d->n_q_heads;
  if (heads_q > 65535 || (d->seq_len + 63) / 64 > 65535) return ULY_ERR_SHAPE;  // grid limits
  if (d->dtype == ULY_F32 && d->head_dim != 64 && d->head_dim != 128) return ULY_ERR_UNSUPPORTED;
  if (d->dtype == ULY_BF16 && d->head_dim != 128) return ULY_ERR_UNSUPPORTED;
  g.B = d->batch;
  g.n = d->seq_len;
  g.P = d->world;
  g.hl = d->n_q_heads / d->world;
  g.gl = d->n_kv_heads / d->world;
  g.group = d->n_q_heads / d->n_kv_heads;
  g.scale = d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / std::sqrt((float)d->head_dim);
  g.out_seq = d->out_seq_layout;
  mk.mask = d->mask;
  mk.n = d->seq_len;
  mk.cu = d->cu_seqlens;
  mk.num_docs = d->num_docs;
  return ULY_OK;
}

// One thread: cu_seqlens must start at 0, never decrease and end at n (the
// pad tail is the last document).  Anything else is reported as
// ULY_ERR_SHAPE in the error word; the attention kernels clamp document
// bounds to the sequence, so a malformed table never sends them outside
// their operands.
__global__ void check_cu_seqlens_kernel(const int32_t *__restrict__ cu, int num_docs, int n, int *err) {
  bool ok = __ldg(cu) == 0 && __ldg(cu + num_docs) == n;
  for (int e = 0; ok && e < num_docs; ++e) ok = __ldg(cu + e) <= __ldg(cu + e + 1);
  if (!ok) raise_error(err, ULY_ERR_SHAPE);
}

uly_status check_cu_seqlens(const uly_attn_desc *d, cudaStream_t s) {
  if (d->mask != ULY_MASK_DOC_CAUSAL) return ULY_OK;
  prof::Scope scope(prof::K_CHECK_CU, s);
  check_cu_seqlens_kernel<<<1, 1, 0, s>>>(d->cu_seqlens, d->num_docs, d->seq_len, error_word());
  note_launches(1);
  return last_launch_status();
}

size_t elem_bytes(int dtype) { return dtype == ULY_BF16 ? 2 : 4; }
size_t q_bytes(const uly_attn_desc *d) {
  return (size_t)d->batch * d->seq_len * d->n_q_heads * d->head_dim * elem_bytes(d->dtype);
}
size_t kv_bytes(const uly_attn_desc *d) {
  return (size_t)d->batch * d->seq_len * d->n_kv_heads * d->head_dim * elem_bytes(d->dtype);
}
size_t lse_bytes(const uly_attn_desc *d) {
  return (size_t)d->batch * d->seq_len * d->n_q_heads * sizeof(float);
}
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool all_aligned(std::initializer_list<const void *> ps) {
  for (const void *p : ps)
    if (!aligned16(p)) return false;
  return true;
}

}  // namespace
}  // namespace uly

using namespace uly;

extern "C" {

uly_status ulysses_seq_to_head(int32_t batch, int32_t seq_len, int32_t world, int32_t heads,
                               int32_t head_dim, int32_t eb, const void *src, void *dst,
                               void *stream) {
  uly_status st = permute_validate(batch, seq_len, world, heads, head_dim, eb, src, dst);
  if (st != ULY_OK) return st;
  return permute_launch(true, batch, seq_len, world, heads, head_dim, eb, src, dst,
                        static_cast<cudaStream_t>(stream));
}

uly_status ulysses_head_to_seq(int32_t batch, int32_t seq_len, int32_t world, int32_t heads,
                               int32_t head_dim, int32_t eb, const void *src, void *dst,
                               void *stream) {
  uly_status st = permute_validate(batch, seq_len, world, heads, head_dim, eb, src, dst);
  if (st != ULY_OK) return st;
  return permute_launch(false, batch, seq_len, world, heads, head_dim, eb, src, dst,
                        static_cast<cudaStream_t>(stream));
}

static uly_status permute_batch(bool to_head, int32_t batch, int32_t seq_len, int32_t world, int32_t head_dim,
                                int32_t eb, int32_t count, const uly_permute_item *items, void *stream) {
  if (!items) return ULY_ERR_NULL;
  if (count < 1 || count > 4) return ULY_ERR_SHAPE;
  size_t bytes[4];
  for (int i = 0; i < count; ++i) {
    uly_status st = permute_validate(batch, seq_len, world, items[i].heads, head_dim, eb, items[i].src,
                                     items[i].dst);
    if (st != ULY_OK) return st;
    bytes[i] = (size_t)batch * seq_len * items[i].heads * head_dim * eb;
  }
  for (int i = 0; i < count; ++i)
    for (int j = 0; j < count; ++j)
      if (i != j && (overlap(items[i].dst, bytes[i], items[j].dst, bytes[j]) ||
                     overlap(items[i].dst, bytes[i], items[j].src, bytes[j])))
        return ULY_ERR_ALIAS;
  return permute_batch_launch(to_head, batch, seq_len, world, head_dim, eb, count, items,
                              static_cast<cudaStream_t>(stream));
}

uly_status ulysses_seq_to_head_batch(int32_t batch, int32_t seq_len, int32_t world, int32_t head_dim,
                                     int32_t eb, int32_t count, const uly_permute_item *items, void *stream) {
  return permute_batch(true, batch, seq_len, world, head_dim, eb, count, items, stream);
}

uly_status ulysses_head_to_seq_batch(int32_t batch, int32_t seq_len, int32_t world, int32_t head_dim,
                                     int32_t eb, int32_t count, const uly_permute_item *items, void *stream) {
  return permute_batch(false, batch, seq_len, world, head_dim, eb, count, items, stream);
}

uly_status ulysses_kv_seq_to_head_replicated(int32_t batch, int32_t seq_len, int32_t world,
                                             int32_t kv_heads, int32_t head_dim, int32_t eb,
                                             const void *src, void *dst, void *stream) {
  uly_status st = kv_rep_validate(batch, seq_len, world, kv_heads, head_dim, eb, src, dst);
  if (st != ULY_OK) return st;
  return kv_replicate_launch(batch, seq_len, world, kv_heads, head_dim, eb, src, dst,
                             static_cast<cudaStream_t>(stream));
}

uly_status ulysses_kv_head_to_seq_reduce(int32_t batch, int32_t seq_len, int32_t world,
                                         int32_t kv_heads, int32_t head_dim, int32_t dtype,
                                         const void *src, void *dst, void *stream) {
  if (dtype != ULY_F32 && dtype != ULY_BF16) return ULY_ERR_DTYPE;
  // the same rules as the forward copy with the roles of the buffers swapped
  // (dst holds the G heads, src the P copies)
  uly_status st = kv_rep_validate(batch, seq_len, world, kv_heads, head_dim,
                                  dtype == ULY_BF16 ? 2 : 4, dst, src);
  if (st != ULY_OK) return st;
  return kv_reduce_launch(batch, seq_len, world, kv_heads, head_dim, dtype, src, dst,
                          static_cast<cudaStream_t>(stream));
}

uly_status ulysses_shift_labels(int32_t batch, int32_t seq_len, int32_t world,
                                const int32_t *input_ids, const int32_t *cu_seqlens,
                                int32_t num_docs, int32_t valid_len, int32_t ignore_index,
                                int32_t *labels, void *stream) {
  if (!input_ids || !labels) return ULY_ERR_NULL;
  if (batch <= 0 || seq_len <= 0 || world <= 0 || seq_len % world) return ULY_ERR_SHAPE;
  if (valid_len < 0 || valid_len > seq_len) return ULY_ERR_SHAPE;
  if (num_docs < 0 || (num_docs > 0 && !cu_seqlens)) return ULY_ERR_NULL;
  if ((long long)batch * seq_len > (1LL << 40)) return ULY_ERR_SHAPE;
  const size_t bytes = (size_t)batch * seq_len * sizeof(int32_t);
  if (overlap(input_ids, bytes, labels, bytes)) return ULY_ERR_ALIAS;
  if (num_docs > 0 && overlap(cu_seqlens, (size_t)(num_docs + 1) * sizeof(int32_t), labels, bytes))
    return ULY_ERR_ALIAS;
  return shift_labels_launch(batch, seq_len, world, input_ids, cu_seqlens, num_docs, valid_len,
                             ignore_index, labels, static_cast<cudaStream_t>(stream));
}

uly_status ulysses_rope_table(int32_t max_pos, int32_t head_dim, double base, float *table,
                              void *stream) {
  if (!table) return ULY_ERR_NULL;
  if (max_pos <= 0 || head_dim <= 0 || head_dim % 2) return ULY_ERR_SHAPE;
  if (!(base > 1.0) || !std::isfinite(base)) return ULY_ERR_SHAPE;
  if ((long long)max_pos * head_dim > (1LL << 40)) return ULY_ERR_SHAPE;
  if (!aligned16(table)) return ULY_ERR_ALIGN;
  return rope_table_launch(max_pos, head_dim, base, table, static_cast<cudaStream_t>(stream));
}

uly_status ulysses_qkv_proj_rope(int32_t batch, int32_t seq_len, int32_t world, int32_t hidden,
                                 int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                 const void *x, const void *w_qkv, const float *rope_table,
                                 int32_t max_pos, const int32_t *positions, void *q, void *k,
                                 void *v, void *stream) {
  if (!x || !w_qkv || !rope_table || !q || !k || !v) return ULY_ERR_NULL;
  if (batch <= 0 || seq_len <= 0 || world <= 0 || hidden <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 ||
      head_dim <= 0 || max_pos <= 0)
    return ULY_ERR_SHAPE;
  if (seq_len % world || n_q_heads % world || n_q_heads % n_kv_heads) return ULY_ERR_SHAPE;
  if (n_kv_heads % world) return ULY_ERR_UNSUPPORTED;  // fewer KV heads than ranks: project, then copy
  if (head_dim != 128 || (n_q_heads + 2 * n_kv_heads) % 2 || hidden % 64) return ULY_ERR_UNSUPPORTED;
  if (!positions && max_pos < seq_len) return ULY_ERR_SHAPE;
  const long long M = (long long)batch * seq_len;
  if ((M + 127) / 128 * ((n_q_heads + 2 * n_kv_heads) / 2) > 0x7fffffffLL) return ULY_ERR_SHAPE;
  if (!all_aligned({x, w_qkv, rope_table, q, k, v})) return ULY_ERR_ALIGN;
  const size_t xb = (size_t)M * hidden * 2, wb = (size_t)(n_q_heads + 2 * n_kv_heads) * head_dim * hidden * 2;
  const size_t qb = (size_t)M * n_q_heads * head_dim * 2, kb = (size_t)M * n_kv_heads * head_dim * 2;
  const size_t rb = (size_t)max_pos * head_dim * 4, pb = positions ? (size_t)M * 4 : 0;
  const void *outs[3] = {q, k, v};
  const size_t osz[3] = {qb, kb, kb};
  for (int i = 0; i < 3; ++i) {
    if (overlap(outs[i], osz[i], x, xb) || overlap(outs[i], osz[i], w_qkv, wb) ||
        overlap(outs[i], osz[i], rope_table, rb) || (positions && overlap(outs[i], osz[i], positions, pb)))
      return ULY_ERR_ALIAS;
    for (int j = i + 1; j < 3; ++j)
      if (overlap(outs[i], osz[i], outs[j], osz[j])) return ULY_ERR_ALIAS;
  }
  return qkv_proj_launch(batch, seq_len, world, hidden, n_q_heads, n_kv_heads, x, w_qkv, rope_table,
                         max_pos, positions, q, k, v, static_cast<cudaStream_t>(stream));
}

uly_status ulysses_o_proj(int32_t batch, int32_t seq_len, int32_t world, int32_t hidden,
                          int32_t n_q_heads, int32_t head_dim, const void *o, const void *w_o,
                          void *y, void *stream) {
  if (!o || !w_o || !y) return ULY_ERR_NULL;
  if (batch <= 0 || seq_len <= 0 || world <= 0 || hidden <= 0 || n_q_heads <= 0 || head_dim <= 0)
    return ULY_ERR_SHAPE;
  if (seq_len % world || n_q_heads % world) return ULY_ERR_SHAPE;
  if (head_dim != 128 || hidden % 256) return ULY_ERR_UNSUPPORTED;
  const long long tiles = (long long)batch * ((seq_len + 127) / 128) * (hidden / 256);
  if (tiles > 0x7fffffffLL || (long long)world * batch * (n_q_heads / world) > 0x7fffffffLL)
    return ULY_ERR_SHAPE;
  if (!all_aligned({o, w_o, y})) return ULY_ERR_ALIGN;
  const size_t ob = (size_t)batch * seq_len * n_q_heads * head_dim * 2;
  const size_t wb = (size_t)hidden * n_q_heads * head_dim * 2, yb = (size_t)batch * seq_len * hidden * 2;
  if (overlap(y, yb, o, ob) || overlap(y, yb, w_o, wb)) return ULY_ERR_ALIAS;
  return o_proj_launch(batch, seq_len, world, hidden, n_q_heads, o, w_o, y,
                       static_cast<cudaStream_t>(stream));
}

uly_status ulysses_qkv_proj_rope_bwd_workspace_size(int32_t batch, int32_t seq_len, int32_t n_q_heads,
                                                   int32_t n_kv_heads, int32_t head_dim, size_t *bytes) {
  if (!bytes) return ULY_ERR_NULL;
  if (batch <= 0 || seq_len <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0) return ULY_ERR_SHAPE;
  *bytes = align256((size_t)batch * seq_len * (n_q_heads + 2 * n_kv_heads) * head_dim * 2);
  return ULY_OK;
}

uly_status ulysses_qkv_proj_rope_bwd(int32_t batch, int32_t seq_len, int32_t world, int32_t hidden,
                                     int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, const void *x,
                                     const void *w_qkv, const float *rope_table, int32_t max_pos,
                                     const int32_t *positions, const void *dq, const void *dk, const void *dv,
                                     void *dx, float *dw, void *workspace, size_t workspace_bytes, void *stream) {
  if (!x || !w_qkv || !rope_table || !dq || !dk || !dv || !dx || !dw) return ULY_ERR_NULL;
  if (batch <= 0 || seq_len <= 0 || world <= 0 || hidden <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 ||
      head_dim <= 0 || max_pos <= 0)
    return ULY_ERR_SHAPE;
  if (seq_len % world || n_q_heads % world || n_q_heads % n_kv_heads) return ULY_ERR_SHAPE;
  if (n_kv_heads % world) return ULY_ERR_UNSUPPORTED;  // fewer KV heads than ranks: sum the copies first
  if (head_dim != 128 || (n_q_heads + 2 * n_kv_heads) % 2 || hidden % 256) return ULY_ERR_UNSUPPORTED;
  if (!positions && max_pos < seq_len) return ULY_ERR_SHAPE;
  const long long M = (long long)batch * seq_len;
  const long long N = (long long)(n_q_heads + 2 * n_kv_heads) * head_dim;
  if (M > 0x7fffffffLL || (M + 127) / 128 * (hidden / 256) > 0x7fffffffLL) return ULY_ERR_SHAPE;
  size_t need = 0;
  ulysses_qkv_proj_rope_bwd_workspace_size(batch, seq_len, n_q_heads, n_kv_heads, head_dim, &need);
  if (!workspace || workspace_bytes < need) return ULY_ERR_WORKSPACE;
  if (!all_aligned({x, w_qkv, rope_table, dq, dk, dv, dx, dw, workspace})) return ULY_ERR_ALIGN;
  const size_t xb = (size_t)M * hidden * 2, wb = (size_t)N * hidden * 2, qb = (size_t)M * n_q_heads * head_dim * 2,
               kb = (size_t)M * n_kv_heads * head_dim * 2, rb = (size_t)max_pos * head_dim * 4,
               pb = positions ? (size_t)M * 4 : 0;
  const void *ins[7] = {x, w_qkv, rope_table, positions, dq, dk, dv};
  const size_t inb[7] = {xb, wb, rb, pb, qb, kb, kb};
  void *outs[3] = {dx, dw, workspace};
  const size_t outb[3] = {xb, (size_t)N * hidden * 4, need};
  for (int a = 0; a < 3; ++a) {
    for (int b = 0; b < 7; ++b)
      if (ins[b] && overlap(outs[a], outb[a], ins[b], inb[b])) return ULY_ERR_ALIAS;
    for (int b = a + 1; b < 3; ++b)
      if (overlap(outs[a], outb[a], outs[b], outb[b])) return ULY_ERR_ALIAS;
  }
  return qkv_proj_bwd_launch(batch, seq_len, world, hidden, n_q_heads, n_kv_heads, x, w_qkv, rope_table, max_pos,
                             positions, dq, dk, dv, dx, dw, workspace, static_cast<cudaStream_t>(stream));
}

uly_status ulysses_o_proj_bwd(int32_t batch, int32_t seq_len, int32_t world, int32_t hidden, int32_t n_q_heads,
                              int32_t head_dim, const void *o_seq, const void *w_o, const void *dy, void *do_head,
                              float *dw_o, void *stream) {
  if (!o_seq || !w_o || !dy || !do_head || !dw_o) return ULY_ERR_NULL;
  if (batch <= 0 || seq_len <= 0 || world <= 0 || hidden <= 0 || n_q_heads <= 0 || head_dim <= 0)
    return ULY_ERR_SHAPE;
  if (seq_len % world || n_q_heads % world) return ULY_ERR_SHAPE;
  if (head_dim != 128 || hidden % 256 || n_q_heads % 2) return ULY_ERR_UNSUPPORTED;
  const long long M = (long long)batch * seq_len;
  if (M > 0x7fffffffLL) return ULY_ERR_SHAPE;
  if (!all_aligned({o_seq, w_o, dy, do_head, dw_o})) return ULY_ERR_ALIGN;
  const size_t ob = (size_t)M * n_q_heads * head_dim * 2, wb = (size_t)hidden * n_q_heads * head_dim * 2,
               yb = (size_t)M * hidden * 2, dwb = (size_t)hidden * n_q_heads * head_dim * 4;
  const void *ins[3] = {o_seq, w_o, dy};
  const size_t inb[3] = {ob, wb, yb};
  for (int b = 0; b < 3; ++b)
    if (overlap(do_head, ob, ins[b], inb[b]) || overlap(dw_o, dwb, ins[b], inb[b])) return ULY_ERR_ALIAS;
  if (overlap(do_head, ob, dw_o, dwb)) return ULY_ERR_ALIAS;
  return o_proj_bwd_launch(batch, seq_len, world, hidden, n_q_heads, o_seq, w_o, dy, do_head, dw_o,
                           static_cast<cudaStream_t>(stream));
}

uly_status ulysses_attn_fwd(const uly_attn_desc *d, const void *q, const void *k, const void *v,
                            void *o, float *lse, void *stream) {
  HeadGeom g;
  MaskInfo mk;
  uly_status st = check_desc(d, g, mk);
  if (st != ULY_OK) return st;
  if (!q || !k || !v || !o || !lse) return ULY_ERR_NULL;
  if (!all_aligned({q, k, v, o, lse})) return ULY_ERR_ALIGN;
  const size_t qb = q_bytes(d), kb = kv_bytes(d), lb = lse_bytes(d);
  for (const void *in : {q, k, v}) {
    const size_t ib = (in == q) ? qb : kb;
    if (overlap(in, ib, o, qb) || overlap(in, ib, lse, lb)) return ULY_ERR_ALIAS;
  }
  if (overlap(o, qb, lse, lb)) return ULY_ERR_ALIAS;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = check_cu_seqlens(d, s)) != ULY_OK) return st;
  if (d->dtype == ULY_F32) return attn_f32_fwd_launch(d, g, mk, q, k, v, o, lse, s);
  return attn_bf16_fwd_launch(d, g, mk, q, k, v, o, lse, s);
}

uly_status ulysses_attn_bwd_workspace_size(const uly_attn_desc *d, size_t *bytes) {
  HeadGeom g;
  MaskInfo mk;
  if (!bytes) return ULY_ERR_NULL;
  uly_status st = check_desc(d, g, mk);
  if (st != ULY_OK) return st;
  if (d->dtype == ULY_BF16) {
    // D_i and LSE_i log2(e), query rows padded per head (+ the fused pass's dQ accumulator)
    *bytes = attn_bf16_bwd_workspace(g, d->deterministic != 0);
  } else {
    *bytes = align256(lse_bytes(d));  // D_i = <dO_i, O_i> for every query row
  }
  return ULY_OK;
}

uly_status ulysses_attn_bwd(const uly_attn_desc *d, const void *q, const void *k, const void *v,
                            const void *o, const float *lse, const void *dout, void *dq, void *dk,
                            void *dv, void *workspace, size_t workspace_bytes, void *stream) {
  HeadGeom g;
  MaskInfo mk;
  uly_status st = check_desc(d, g, mk);
  if (st != ULY_OK) return st;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return ULY_ERR_NULL;
  size_t need = 0;
  ulysses_attn_bwd_workspace_size(d, &need);
  if (!workspace || workspace_bytes < need) return ULY_ERR_WORKSPACE;
  if (!all_aligned({q, k, v, o, lse, dout, dq, dk, dv, workspace})) return ULY_ERR_ALIGN;
  const size_t qb = q_bytes(d), kb = kv_bytes(d), lb = lse_bytes(d);
  const void *ins[6] = {q, k, v, o, lse, dout};
  const size_t inb[6] = {qb, kb, kb, qb, lb, qb};
  void *outs[4] = {dq, dk, dv, workspace};
  const size_t outb[4] = {qb, kb, kb, need};
  for (int a = 0; a < 4; ++a) {
    for (int b = 0; b < 6; ++b)
      if (overlap(outs[a], outb[a], ins[b], inb[b])) return ULY_ERR_ALIAS;
    for (int b = a + 1; b < 4; ++b)
      if (overlap(outs[a], outb[a], outs[b], outb[b])) return ULY_ERR_ALIAS;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = check_cu_seqlens(d, s)) != ULY_OK) return st;
  float *Dv = static_cast<float *>(workspace);
  if (d->dtype == ULY_F32)
    return attn_f32_bwd_launch(d, g, mk, q, k, v, o, lse, dout, dq, dk, dv, Dv, s);
  return attn_bf16_bwd_launch(d, g, mk, q, k, v, o, lse, dout, dq, dk, dv, Dv, s);
}

uly_status ulysses_loss_workspace_size(int32_t world, int64_t tokens, int32_t vocab, size_t *bytes) {
  if (!bytes) return ULY_ERR_NULL;
  if (world <= 0 || tokens < 0 || vocab <= 0 || tokens % world) return ULY_ERR_SHAPE;
  *bytes = align256(loss_workspace_bytes(world, tokens / world));
  return ULY_OK;
}

uly_status ulysses_loss_aggregate(int32_t world, int64_t tokens, int32_t vocab, int32_t logit_dtype,
                                  const void *logits, const int32_t *labels, int32_t ignore_index,
                                  float *shard_sum, int64_t *shard_count, float *loss,
                                  void *workspace, size_t workspace_bytes, void *stream) {
  uly_status st = loss_validate(world, tokens, vocab, logit_dtype, logits, labels, shard_sum,
                                shard_count, loss);
  if (st != ULY_OK) return st;
  size_t need = 0;
  ulysses_loss_workspace_size(world, tokens, vocab, &need);
  if (!workspace || workspace_bytes < need) return ULY_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ULY_ERR_ALIGN;
  const size_t zb = (size_t)tokens * vocab * (logit_dtype == ULY_BF16 ? 2 : 4);
  const size_t yb = (size_t)tokens * 4;
  const void *outs[4] = {shard_sum, shard_count, loss, workspace};
  const size_t outb[4] = {(size_t)world * 4, (size_t)world * 8, 4, need};
  for (int a = 0; a < 4; ++a)
    if (overlap(outs[a], outb[a], logits, zb) || overlap(outs[a], outb[a], labels, yb))
      return ULY_ERR_ALIAS;
  return loss_launch(world, tokens, vocab, logit_dtype, logits, labels, ignore_index, shard_sum,
                     shard_count, loss, workspace, static_cast<cudaStream_t>(stream));
}

uly_status ulysses_loss_bwd_workspace_size(int32_t world, int64_t tokens, int32_t vocab, size_t *bytes) {
  if (!bytes) return ULY_ERR_NULL;
  if (world <= 0 || tokens < 0 || vocab <= 0 || tokens % world) return ULY_ERR_SHAPE;
  *bytes = align256(loss_bwd_workspace_bytes(world, tokens / world));
  return ULY_OK;
}

uly_status ulysses_loss_aggregate_bwd(int32_t world, int64_t tokens, int32_t vocab, int32_t logit_dtype,
                                      const void *logits, const int32_t *labels, int32_t ignore_index,
                                      void *dlogits, float *shard_sum, int64_t *shard_count, float *loss,
                                      void *workspace, size_t workspace_bytes, void *stream) {
  uly_status st = loss_validate(world, tokens, vocab, logit_dtype, logits, labels, shard_sum,
                                shard_count, loss);
  if (st != ULY_OK) return st;
  if (!dlogits) return ULY_ERR_NULL;
  if (!aligned16(dlogits)) return ULY_ERR_ALIGN;
  size_t need = 0;
  ulysses_loss_bwd_workspace_size(world, tokens, vocab, &need);
  if (!workspace || workspace_bytes < need) return ULY_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ULY_ERR_ALIGN;
  const size_t zb = (size_t)tokens * vocab * (logit_dtype == ULY_BF16 ? 2 : 4);
  const size_t yb = (size_t)tokens * 4;
  const void *outs[5] = {dlogits, shard_sum, shard_count, loss, workspace};
  const size_t outb[5] = {zb, (size_t)world * 4, (size_t)world * 8, 4, need};
  for (int a = 0; a < 5; ++a) {
    if (overlap(outs[a], outb[a], logits, zb) || overlap(outs[a], outb[a], labels, yb))
      return ULY_ERR_ALIAS;
    for (int b = a + 1; b < 5; ++b)
      if (overlap(outs[a], outb[a], outs[b], outb[b])) return ULY_ERR_ALIAS;
  }
  return loss_bwd_launch(world, tokens, vocab, logit_dtype, logits, labels, ignore_index, dlogits,
                         shard_sum, shard_count, loss, workspace, static_cast<cudaStream_t>(stream));
}

uly_status ulysses_read_error_info(int32_t *info, int32_t n) {
  if (!info) return ULY_ERR_NULL;
  if (n < 1) return ULY_ERR_SHAPE;
  int *p = error_word();
  if (!p) return ULY_ERR_CUDA;
  int host[kErrInfoWords] = {0}, zero[kErrInfoWords] = {0};
  if (cudaDeviceSynchronize() != cudaSuccess) return ULY_ERR_CUDA;
  if (cudaMemcpy(host, p, sizeof(host), cudaMemcpyDeviceToHost) != cudaSuccess) return ULY_ERR_CUDA;
  if (cudaMemcpy(p, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return ULY_ERR_CUDA;
  for (int i = 0; i < n; ++i) info[i] = i < kErrInfoWords ? host[i] : 0;
  return ULY_OK;
}

uly_status ulysses_error_word(int32_t **dev_word) {
  if (!dev_word) return ULY_ERR_NULL;
  int *p = error_word();
  if (!p) return ULY_ERR_CUDA;
  *dev_word = p;
  return ULY_OK;
}

uly_status ulysses_set_wait_limit(int64_t cycles) {
  if (cycles < 0) return ULY_ERR_SHAPE;
  g_wait_limit.store(cycles == 0 || cycles > kDefaultWaitLimit ? kDefaultWaitLimit : cycles,
                     std::memory_order_relaxed);
  return ULY_OK;
}

uly_status ulysses_set_attn_block_order(int32_t order) {
  if (order != ULY_BLOCK_ORDER_AUTO && order != ULY_BLOCK_ORDER_KV_HEAD_MAJOR &&
      order != ULY_BLOCK_ORDER_HEAVIEST_FIRST)
    return ULY_ERR_SHAPE;
  g_attn_block_order.store(order, std::memory_order_relaxed);
  return ULY_OK;
}

uly_status ulysses_read_error(int32_t *word) {
  if (!word) return ULY_ERR_NULL;
  return ulysses_read_error_info(word, 1);
}

const char *ulysses_status_string(uly_status s) {
  switch (s) {
    case ULY_OK: return "ok";
    case ULY_ERR_NULL: return "null pointer";
    case ULY_ERR_SHAPE: return "invalid shape";
    case ULY_ERR_DTYPE: return "invalid dtype";
    case ULY_ERR_ALIGN: return "misaligned pointer or row";
    case ULY_ERR_ALIAS: return "input and output overlap";
    case ULY_ERR_UNSUPPORTED: return "unsupported configuration";
    case ULY_ERR_CUDA: return "CUDA runtime error";
    case ULY_ERR_LABEL: return "label out of range";
    case ULY_ERR_TIMEOUT: return "bounded wait timed out";
    case ULY_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

uint64_t ulysses_launch_count(void) { return g_launches.load(); }

}  // extern "C"
