// The all-to-alls of K and V when there are fewer KV heads than ranks
// (G < P, P % G == 0): the copying seq -> head redistribution and, for the
// gradients, the summing head -> seq reverse.  Byte / vector copies, HBM-bound.
#include "common.cuh"
#include "prof.cuh"

namespace uly {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 8;  // 16-byte vectors in flight per thread

// KV heads fewer than ranks (G < P, P % G == 0).  Every rank needs the one
// KV head its query heads use -- rank r2 uses KV head floor(r2*G/P) -- so the
// first all-to-all sends each KV head whole to its rep = P/G using ranks
// ("Ulysses 序列平行化", section "與 Ring Attention 的比較": the method needs
// at least as many heads as ranks; grouped KV heads are copied to meet it).
//   seq layout  X[r][b][tt][k][:]      k < G
//   head layout Y[r2][b][0][t][:]      t = r*s + tt, one KV head per rank
// A CTA reads one contiguous block of TOK*G source rows once and writes each
// row to its rep destinations.
template <int VPR>
__global__ void __launch_bounds__(kThreads) kv_replicate_kernel(
    const uint4 *__restrict__ src, uint4 *__restrict__ dst, int B, int n, int s, int G, int rep,
    int tok_per_cta) {
  const int rb = blockIdx.y;  // sending rank r and batch b
  const int r = rb / B, b = rb - r * B;
  const int tt0 = blockIdx.x * tok_per_cta;
  const int ntok = min(tok_per_cta, s - tt0);
  if (ntok <= 0) return;
  const long long total = (long long)ntok * G * VPR;
  const long long seq_row0 = ((long long)rb * s + tt0) * G;
  for (long long base = (long long)threadIdx.x; base < total; base += (long long)kThreads * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long e = base + (long long)u * kThreads;
      if (e < total) v[u] = __ldcs(src + seq_row0 * VPR + e);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long e = base + (long long)u * kThreads;
      if (e < total) {
        const int row = (int)(e / VPR), lane = (int)(e % VPR);
        const int tok = row / G, k = row - tok * G;
        const long long t = (long long)r * s + tt0 + tok;
        for (int j = 0; j < rep; ++j) {
          const long long r2 = (long long)k * rep + j;
          __stcs(dst + ((r2 * B + b) * n + t) * VPR + lane, v[u]);
        }
      }
    }
  }
}

__device__ __forceinline__ void add_vec(float (&acc)[8], const uint4 &v, bool bf16) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if (bf16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += __uint_as_float(w[i] << 16);
      acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] += __uint_as_float(w[i]);
  }
}

__device__ __forceinline__ uint4 pack_acc(const float (&acc)[8], bool bf16) {
  if (!bf16) return make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]),
                               __float_as_uint(acc[2]), __float_as_uint(acc[3]));
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i]));
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i + 1]));
    w[i] = lo | (hi << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Reverse of kv_replicate_kernel for gradients: a KV head's gradient is the
// sum of what its rep copies received, summed in fp32 in rank order and
// rounded once to the element type.  A CTA writes one contiguous block of
// TOK*G destination rows (seq layout of rank r); each 16-byte vector reads its
// rep source vectors (one per copy), all in flight together.
template <int VPR, bool BF16>
__global__ void __launch_bounds__(kThreads) kv_reduce_kernel(
    const uint4 *__restrict__ src, uint4 *__restrict__ dst, int B, int n, int s, int G, int rep,
    int tok_per_cta) {
  constexpr int kU = 4;
  const int rb = blockIdx.y;  // receiving rank r and batch b
  const int r = rb / B, b = rb - r * B;
  const int tt0 = blockIdx.x * tok_per_cta;
  const int ntok = min(tok_per_cta, s - tt0);
  if (ntok <= 0) return;
  const long long total = (long long)ntok * G * VPR;
  const long long seq_row0 = ((long long)rb * s + tt0) * G;
  for (long long base = (long long)threadIdx.x; base < total; base += (long long)kThreads * kU) {
    float acc[kU][8];
    long long srcv[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
      const long long e = base + (long long)u * kThreads;
      srcv[u] = -1;
      if (e < total) {
        const int row = (int)(e / VPR), lane = (int)(e % VPR);
        const int tok = row / G, k = row - tok * G;
        const long long t = (long long)r * s + tt0 + tok;
        srcv[u] = (((long long)k * rep * B + b) * n + t) * VPR + lane;  // copy j = 0
      }
    }
    const long long copy_stride = (long long)B * n * VPR;  // next rank's copy
    for (int j = 0; j < rep; ++j) {
      uint4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (srcv[u] >= 0) v[u] = __ldcs(src + srcv[u] + (long long)j * copy_stride);
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (srcv[u] >= 0) add_vec(acc[u], v[u], BF16);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const long long e = base + (long long)u * kThreads;
      if (e < total) __stcs(dst + seq_row0 * VPR + e, pack_acc(acc[u], BF16));
    }
  }
}

int kv_tok_per_cta(int G, int vpr, int s) {
  int tok = 4096 / (G * vpr);
  if (tok < 1) tok = 1;
  if (tok > s) tok = s;
  return tok;
}

}  // namespace

uly_status kv_rep_validate(int32_t B, int32_t n, int32_t P, int32_t G, int32_t d, int32_t elem_bytes,
                           const void *src, const void *dst) {
  if (!src || !dst) return ULY_ERR_NULL;
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8) return ULY_ERR_DTYPE;
  if (B <= 0 || n <= 0 || P <= 0 || G <= 0 || d <= 0) return ULY_ERR_SHAPE;
  if (n % P || P % G) return ULY_ERR_SHAPE;
  if (B > 65535 / P) return ULY_ERR_SHAPE;
  const long long row = (long long)d * elem_bytes;
  if (row % 16) return ULY_ERR_ALIGN;
  const long long vpr = row / 16;
  if (vpr > 64 || (vpr & (vpr - 1))) return ULY_ERR_UNSUPPORTED;
  if (!aligned16(src) || !aligned16(dst)) return ULY_ERR_ALIGN;
  const size_t in_bytes = (size_t)B * n * G * row, out_bytes = (size_t)B * n * P * row;
  if (overlap(src, in_bytes, dst, out_bytes)) return ULY_ERR_ALIAS;
  return ULY_OK;
}

uly_status kv_replicate_launch(int32_t B, int32_t n, int32_t P, int32_t G, int32_t d, int32_t eb,
                               const void *src, void *dst, cudaStream_t stream) {
  const int vpr = (int)((long long)d * eb / 16), s = n / P, rep = P / G;
  const int tok = kv_tok_per_cta(G, vpr, s);
  dim3 grid((s + tok - 1) / tok, P * B);
  const uint4 *in = static_cast<const uint4 *>(src);
  uint4 *out = static_cast<uint4 *>(dst);
  prof::Scope scope(prof::K_KV_REPLICATE, stream);
#define ULY_REP_CASE(V)                                                                        \
  case V:                                                                                      \
    kv_replicate_kernel<V><<<grid, kThreads, 0, stream>>>(in, out, B, n, s, G, rep, tok);      \
    break;
  switch (vpr) {
    ULY_REP_CASE(1)
    ULY_REP_CASE(2)
    ULY_REP_CASE(4)
    ULY_REP_CASE(8)
    ULY_REP_CASE(16)
    ULY_REP_CASE(32)
    ULY_REP_CASE(64)
    default:
      return ULY_ERR_UNSUPPORTED;
  }
#undef ULY_REP_CASE
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? ULY_OK : ULY_ERR_CUDA;
}

uly_status kv_reduce_launch(int32_t B, int32_t n, int32_t P, int32_t G, int32_t d, int32_t dtype,
                            const void *src, void *dst, cudaStream_t stream) {
  const int eb = dtype == ULY_BF16 ? 2 : 4;
  const int vpr = (int)((long long)d * eb / 16), s = n / P, rep = P / G;
  const int tok = kv_tok_per_cta(G, vpr, s);
  dim3 grid((s + tok - 1) / tok, P * B);
  const uint4 *in = static_cast<const uint4 *>(src);
  uint4 *out = static_cast<uint4 *>(dst);
  prof::Scope scope(prof::K_KV_REDUCE, stream);
#define ULY_RED_CASE(V)                                                                          \
  case V:                                                                                        \
    if (dtype == ULY_BF16)                                                                       \
      kv_reduce_kernel<V, true><<<grid, kThreads, 0, stream>>>(in, out, B, n, s, G, rep, tok);   \
    else                                                                                         \
      kv_reduce_kernel<V, false><<<grid, kThreads, 0, stream>>>(in, out, B, n, s, G, rep, tok);  \
    break;
  switch (vpr) {
    ULY_RED_CASE(1)
    ULY_RED_CASE(2)
    ULY_RED_CASE(4)
    ULY_RED_CASE(8)
    ULY_RED_CASE(16)
    ULY_RED_CASE(32)
    ULY_RED_CASE(64)
    default:
      return ULY_ERR_UNSUPPORTED;
  }
#undef ULY_RED_CASE
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? ULY_OK : ULY_ERR_CUDA;
}

}  // namespace uly
