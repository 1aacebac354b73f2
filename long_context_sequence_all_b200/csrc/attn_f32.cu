// Local attention of every logical rank (Ulysses step 4, "Paralelismul de
// Secvență Ulysses", section "Mecanismul de funcționare Ulysses"; standard
// scaled-dot-product attention) in exact fp32 on the CUDA cores.
//
// Tensor cores have no fp32-in / fp32-exact mode (tf32 keeps 10 mantissa
// bits), so the fp32 workload runs here: FFMA dot products, online softmax
// with accurate expf.  Layout: head layout q,o [P][B][H/P][n][d],
// k,v [P][B][G/P][n][d], lse [P][B][H/P][n].
//
// Forward: a CTA owns 64 query rows of one query head; four threads share a
// row (each holds d/4 of q and of the output accumulator) and reduce partial
// dot products with two shuffles.  K/V tiles of 32 keys are staged in shared
// memory.  Backward: D_i = <dO_i, O_i>; a dQ kernel with the same row
// ownership, and a dK/dV kernel that owns 64 keys of one KV head and loops
// over the query rows of every query head of its group (deterministic, no
// atomics).
#include "common.cuh"
#include "prof.cuh"

namespace uly {

namespace {

constexpr int kRows = 64;     // query rows (or key rows) per CTA
constexpr int kTile = 32;     // keys (or query rows) per shared-memory tile
constexpr int kThreads = 256; // 64 rows x 4 threads

__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

template <int D>
__global__ void __launch_bounds__(kThreads) attn_fwd_f32_kernel(
    const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
    float *__restrict__ o, float *__restrict__ lse, HeadGeom g, MaskInfo mk) {
  constexpr int DQ = D / 4;
  __shared__ __align__(16) float Ks[kTile][D];
  __shared__ __align__(16) float Vs[kTile][D];
  const int qh = blockIdx.y;                       // ((r*B + b)*hl + hh)
  const int hh = qh % g.hl, rb = qh / g.hl;
  const int kh = rb * g.gl + hh / g.group;         // KV head of this query head
  const int m0 = blockIdx.x * kRows;
  const int row = threadIdx.x >> 2, part = threadIdx.x & 3;
  const int i = m0 + row;
  const bool valid = i < g.n;
  const float *qrow = q + ((long long)qh * g.n + (valid ? i : 0)) * D + part * DQ;
  float qr[DQ], acc[DQ];
#pragma unroll
  for (int x = 0; x < DQ; ++x) { qr[x] = valid ? qrow[x] : 0.f; acc[x] = 0.f; }
  int lo = 0, hi = -1;
  if (valid) mk.row_range(i, lo, hi);
  int blo, bhi, tmp;
  mk.row_range(m0, blo, tmp);
  mk.row_range(min(m0 + kRows - 1, g.n - 1), tmp, bhi);
  float m = -INFINITY, l = 0.f;
  const float *kb = k + (long long)kh * g.n * D;
  const float *vb = v + (long long)kh * g.n * D;
  for (int j0 = (blo / kTile) * kTile; j0 <= bhi; j0 += kTile) {
    __syncthreads();
    for (int e = threadIdx.x; e < kTile * D / 4; e += kThreads) {
      const int jj = e / (D / 4), c = e % (D / 4);
      const int j = j0 + jj;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (j < g.n) {
        kv = reinterpret_cast<const float4 *>(kb + (long long)j * D)[c];
        vv = reinterpret_cast<const float4 *>(vb + (long long)j * D)[c];
      }
      reinterpret_cast<float4 *>(&Ks[jj][0])[c] = kv;
      reinterpret_cast<float4 *>(&Vs[jj][0])[c] = vv;
    }
    __syncthreads();
    float s[kTile];
    float tmax = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < kTile; ++jj) {
      float p = 0.f;
#pragma unroll
      for (int x = 0; x < DQ; ++x) p = fmaf(qr[x], Ks[jj][part * DQ + x], p);
      p = quad_sum(p) * g.scale;
      const int j = j0 + jj;
      s[jj] = (j >= lo && j <= hi) ? p : -INFINITY;
      tmax = fmaxf(tmax, s[jj]);
    }
    const float mn = fmaxf(m, tmax);
    if (mn == -INFINITY) continue;  // nothing visible yet
    const float alpha = expf(m - mn);  // m = -inf -> 0
    l *= alpha;
#pragma unroll
    for (int x = 0; x < DQ; ++x) acc[x] *= alpha;
    m = mn;
#pragma unroll
    for (int jj = 0; jj < kTile; ++jj) {
      const float p = expf(s[jj] - m);
      l += p;
#pragma unroll
      for (int x = 0; x < DQ; ++x) acc[x] = fmaf(p, Vs[jj][part * DQ + x], acc[x]);
    }
  }
  if (valid) {
    float *orow = o + g.q_out_row(qh, i) * D + part * DQ;
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
    for (int x = 0; x < DQ; ++x) orow[x] = acc[x] * inv;
    if (part == 0) lse[(long long)qh * g.n + i] = (l > 0.f) ? m + logf(l) : -INFINITY;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) attn_dq_f32_kernel(
    const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
    const float *__restrict__ dout, const float *__restrict__ lse, const float *__restrict__ Dv,
    float *__restrict__ dq, HeadGeom g, MaskInfo mk) {
  constexpr int DQ = D / 4;
  __shared__ __align__(16) float Ks[kTile][D];
  __shared__ __align__(16) float Vs[kTile][D];
  const int qh = blockIdx.y;
  const int hh = qh % g.hl, rb = qh / g.hl;
  const int kh = rb * g.gl + hh / g.group;
  const int m0 = blockIdx.x * kRows;
  const int row = threadIdx.x >> 2, part = threadIdx.x & 3;
  const int i = m0 + row;
  const bool valid = i < g.n;
  const long long ro = ((long long)qh * g.n + (valid ? i : 0));
  float qr[DQ], dor[DQ], acc[DQ];
#pragma unroll
  for (int x = 0; x < DQ; ++x) {
    qr[x] = valid ? q[ro * D + part * DQ + x] : 0.f;
    dor[x] = valid ? dout[ro * D + part * DQ + x] : 0.f;
    acc[x] = 0.f;
  }
  const float li = valid ? lse[ro] : 0.f, Di = valid ? Dv[ro] : 0.f;
  int lo = 0, hi = -1;
  if (valid) mk.row_range(i, lo, hi);
  int blo, bhi, tmp;
  mk.row_range(m0, blo, tmp);
  mk.row_range(min(m0 + kRows - 1, g.n - 1), tmp, bhi);
  const float *kb = k + (long long)kh * g.n * D;
  const float *vb = v + (long long)kh * g.n * D;
  for (int j0 = (blo / kTile) * kTile; j0 <= bhi; j0 += kTile) {
    __syncthreads();
    for (int e = threadIdx.x; e < kTile * D / 4; e += kThreads) {
      const int jj = e / (D / 4), c = e % (D / 4);
      const int j = j0 + jj;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (j < g.n) {
        kv = reinterpret_cast<const float4 *>(kb + (long long)j * D)[c];
        vv = reinterpret_cast<const float4 *>(vb + (long long)j * D)[c];
      }
      reinterpret_cast<float4 *>(&Ks[jj][0])[c] = kv;
      reinterpret_cast<float4 *>(&Vs[jj][0])[c] = vv;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < kTile; ++jj) {
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int x = 0; x < DQ; ++x) {
        s = fmaf(qr[x], Ks[jj][part * DQ + x], s);
        dp = fmaf(dor[x], Vs[jj][part * DQ + x], dp);
      }
      s = quad_sum(s) * g.scale;
      dp = quad_sum(dp);
      const int j = j0 + jj;
      const float p = (j >= lo && j <= hi) ? expf(s - li) : 0.f;
      const float ds = p * (dp - Di);
#pragma unroll
      for (int x = 0; x < DQ; ++x) acc[x] = fmaf(ds, Ks[jj][part * DQ + x], acc[x]);
    }
  }
  if (valid) {
#pragma unroll
    const long long out = g.q_out_row(qh, i);
#pragma unroll
    for (int x = 0; x < DQ; ++x) dq[out * D + part * DQ + x] = acc[x] * g.scale;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) attn_dkdv_f32_kernel(
    const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
    const float *__restrict__ dout, const float *__restrict__ lse, const float *__restrict__ Dv,
    float *__restrict__ dk, float *__restrict__ dvv, HeadGeom g, MaskInfo mk) {
  constexpr int DQ = D / 4;
  __shared__ __align__(16) float Qs[kTile][D];
  __shared__ __align__(16) float Os[kTile][D];   // dO tile
  __shared__ float Ls[kTile], Ds[kTile];
  const int kh = blockIdx.y;                     // ((r*B + b)*gl + gg)
  const int gg = kh % g.gl, rb = kh / g.gl;
  const int n0 = blockIdx.x * kRows;
  const int row = threadIdx.x >> 2, part = threadIdx.x & 3;
  const int j = n0 + row;
  const bool valid = j < g.n;
  const long long ko = (long long)kh * g.n + (valid ? j : 0);
  float kr[DQ], vr[DQ], ak[DQ], av[DQ];
#pragma unroll
  for (int x = 0; x < DQ; ++x) {
    kr[x] = valid ? k[ko * D + part * DQ + x] : 0.f;
    vr[x] = valid ? v[ko * D + part * DQ + x] : 0.f;
    ak[x] = 0.f;
    av[x] = 0.f;
  }
  int lo = 0, hi = -1;  // query rows that see key j
  if (valid) mk.col_range(j, lo, hi);
  int blo, bhi, tmp;
  mk.col_range(n0, blo, tmp);
  mk.col_range(min(n0 + kRows - 1, g.n - 1), tmp, bhi);
  for (int e2 = 0; e2 < g.group; ++e2) {
    const int qh = rb * g.hl + gg * g.group + e2;
    const float *qb = q + (long long)qh * g.n * D;
    const float *ob = dout + (long long)qh * g.n * D;
    for (int i0 = (blo / kTile) * kTile; i0 <= bhi; i0 += kTile) {
      __syncthreads();
      for (int e = threadIdx.x; e < kTile * D / 4; e += kThreads) {
        const int ii = e / (D / 4), c = e % (D / 4);
        const int i = i0 + ii;
        float4 qv = make_float4(0.f, 0.f, 0.f, 0.f), ov = qv;
        if (i < g.n) {
          qv = reinterpret_cast<const float4 *>(qb + (long long)i * D)[c];
          ov = reinterpret_cast<const float4 *>(ob + (long long)i * D)[c];
        }
        reinterpret_cast<float4 *>(&Qs[ii][0])[c] = qv;
        reinterpret_cast<float4 *>(&Os[ii][0])[c] = ov;
      }
      if (threadIdx.x < kTile) {
        const int i = i0 + threadIdx.x;
        Ls[threadIdx.x] = i < g.n ? lse[(long long)qh * g.n + i] : 0.f;
        Ds[threadIdx.x] = i < g.n ? Dv[(long long)qh * g.n + i] : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int ii = 0; ii < kTile; ++ii) {
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int x = 0; x < DQ; ++x) {
          s = fmaf(Qs[ii][part * DQ + x], kr[x], s);
          dp = fmaf(Os[ii][part * DQ + x], vr[x], dp);
        }
        s = quad_sum(s) * g.scale;
        dp = quad_sum(dp);
        const int i = i0 + ii;
        const float p = (i >= lo && i <= hi) ? expf(s - Ls[ii]) : 0.f;
        const float ds = p * (dp - Ds[ii]);
#pragma unroll
        for (int x = 0; x < DQ; ++x) {
          av[x] = fmaf(p, Os[ii][part * DQ + x], av[x]);
          ak[x] = fmaf(ds, Qs[ii][part * DQ + x], ak[x]);
        }
      }
    }
  }
  if (valid) {
    const long long out = g.kv_out_row(kh, j);
#pragma unroll
    for (int x = 0; x < DQ; ++x) {
      dk[out * D + part * DQ + x] = ak[x] * g.scale;
      dvv[out * D + part * DQ + x] = av[x];
    }
  }
}

// D_i = <dO_i, O_i> (fp32 path), one warp per row; dout in the head layout,
// O in the head or (g.out_seq) the seq layout.
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_bwd_dot_kernel(const T *__restrict__ o,
                                                           const T *__restrict__ dout,
                                                           float *__restrict__ Dv, long long rows, HeadGeom g) {
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const long long h = r / g.n;
  const long long ro = g.q_out_row(h, (int)(r - h * g.n));
  float acc = 0.f;
  for (int x = lane; x < D; x += 32)
    acc = fmaf(static_cast<float>(o[ro * D + x]), static_cast<float>(dout[r * D + x]), acc);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) Dv[r] = acc;
}

}  // namespace

uly_status attn_f32_fwd_launch(const uly_attn_desc *d, const HeadGeom &g, const MaskInfo &mk,
                               const void *q, const void *k, const void *v, void *o, float *lse,
                               cudaStream_t stream) {
  dim3 grid((g.n + kRows - 1) / kRows, g.P * g.B * g.hl);
  const float *Q = static_cast<const float *>(q), *K = static_cast<const float *>(k),
              *V = static_cast<const float *>(v);
  float *O = static_cast<float *>(o);
  prof::Scope scope(prof::K_ATTN_FWD_F32, stream);
  if (d->head_dim == 64)
    attn_fwd_f32_kernel<64><<<grid, kThreads, 0, stream>>>(Q, K, V, O, lse, g, mk);
  else if (d->head_dim == 128)
    attn_fwd_f32_kernel<128><<<grid, kThreads, 0, stream>>>(Q, K, V, O, lse, g, mk);
  else
    return ULY_ERR_UNSUPPORTED;
  note_launches(1);
  return last_launch_status();
}

uly_status attn_bwd_dot_launch(int dtype, int head_dim, const void *o, const void *dout, float *Dv,
                               long long rows, const HeadGeom &g, cudaStream_t stream) {
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  if (blocks == 0) return ULY_OK;
  prof::Scope scope(prof::K_ATTN_BWD_DOT, stream);
  if (dtype == ULY_F32 && head_dim == 64)
    attn_bwd_dot_kernel<float, 64><<<blocks, 256, 0, stream>>>(
        static_cast<const float *>(o), static_cast<const float *>(dout), Dv, rows, g);
  else if (dtype == ULY_F32 && head_dim == 128)
    attn_bwd_dot_kernel<float, 128><<<blocks, 256, 0, stream>>>(
        static_cast<const float *>(o), static_cast<const float *>(dout), Dv, rows, g);
  else
    return ULY_ERR_UNSUPPORTED;
  note_launches(1);
  return last_launch_status();
}

uly_status attn_f32_bwd_launch(const uly_attn_desc *d, const HeadGeom &g, const MaskInfo &mk,
                               const void *q, const void *k, const void *v, const void *o,
                               const float *lse, const void *dout, void *dq, void *dk, void *dv,
                               float *Dv, cudaStream_t stream) {
  const long long qrows = (long long)g.P * g.B * g.hl * g.n;
  uly_status st = attn_bwd_dot_launch(ULY_F32, d->head_dim, o, dout, Dv, qrows, g, stream);
  if (st != ULY_OK) return st;
  const float *Q = static_cast<const float *>(q), *K = static_cast<const float *>(k),
              *V = static_cast<const float *>(v), *dO = static_cast<const float *>(dout);
  float *dQ = static_cast<float *>(dq), *dK = static_cast<float *>(dk), *dV = static_cast<float *>(dv);
  dim3 gq((g.n + kRows - 1) / kRows, g.P * g.B * g.hl);
  dim3 gk((g.n + kRows - 1) / kRows, g.P * g.B * g.gl);
  if (d->head_dim != 64 && d->head_dim != 128) return ULY_ERR_UNSUPPORTED;
  {
    prof::Scope scope(prof::K_ATTN_DQ_F32, stream);
    if (d->head_dim == 64)
      attn_dq_f32_kernel<64><<<gq, kThreads, 0, stream>>>(Q, K, V, dO, lse, Dv, dQ, g, mk);
    else
      attn_dq_f32_kernel<128><<<gq, kThreads, 0, stream>>>(Q, K, V, dO, lse, Dv, dQ, g, mk);
  }
  {
    prof::Scope scope(prof::K_ATTN_DKDV_F32, stream);
    if (d->head_dim == 64)
      attn_dkdv_f32_kernel<64><<<gk, kThreads, 0, stream>>>(Q, K, V, dO, lse, Dv, dK, dV, g, mk);
    else
      attn_dkdv_f32_kernel<128><<<gk, kThreads, 0, stream>>>(Q, K, V, dO, lse, Dv, dK, dV, g, mk);
  }
  note_launches(2);
  return last_launch_status();
}

}  // namespace uly
