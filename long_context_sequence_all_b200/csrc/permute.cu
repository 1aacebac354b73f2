// The two Ulysses all-to-alls, held inside one GPU's HBM as layout
// permutations ("Paralelismul de Secvență Ulysses", section "Mecanismul de
// funcționare Ulysses", steps 3 and 5):
//
//   seq layout  X[r][b][tt][hg][:]   (rank r holds positions t = r*s + tt)
//   head layout X[r2][b][hh][t][:]   (rank r2 holds heads hg = r2*hl + hh)
//
// Both directions move whole rows of head_dim elements, so the kernel is a
// byte copy of 16-byte vectors: bit-exact for any element type.  A CTA owns
// a run of TOK consecutive tokens of one (rank, batch) pair: on the seq side
// that run is one contiguous block of TOK * heads rows; on the head side it is
// `heads` contiguous runs of TOK rows.  Both sides are therefore read and
// written in full 16-byte vectors by consecutive lanes (coalesced), and all
// index arithmetic is per row, never per byte.
#include "common.cuh"
#include "prof.cuh"

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
  prof::Scope scope(TO_HEAD ? prof::K_SEQ_TO_HEAD : prof::K_HEAD_TO_SEQ, stream);
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

}  // namespace

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

uly_status permute_launch(bool to_head, int32_t B, int32_t n, int32_t P, int32_t heads, int32_t d,
                          int32_t elem_bytes, const void *src, void *dst, cudaStream_t stream) {
  const int vpr = (int)((long long)d * elem_bytes / 16);
  cudaError_t e = to_head ? launch_permute<true>(B, n, P, heads, vpr, src, dst, stream)
                          : launch_permute<false>(B, n, P, heads, vpr, src, dst, stream);
  return e == cudaSuccess ? ULY_OK : ULY_ERR_CUDA;
}

}  // namespace uly
