// Token-weighted cross-entropy aggregated over the P logical ranks
// ("Paralelismul de Secvență Ulysses", section "Integrarea cu Accelerate":
// each rank's loss is weighted by its number of valid tokens, so padding and
// masked prompt tokens do not bias the mean).
//
//   l_t = logsumexp(z_t) - z_t[y_t]          (tokens with y_t != ignore_index)
//   S_r = sum_{t in shard r} l_t,  C_r = #valid tokens of shard r
//   L   = sum_r S_r / sum_r C_r
//
// Pass 1: one warp per token streams the token's logits row once (16-byte
// loads, eight in flight per lane), keeping a running (max, sum) per lane
// (the maximum taken, and the sum rescaled, once per group of eight loaded
// vectors); lanes merge with shuffles.  Every CTA writes one (sum, count) partial for
// its shard into the workspace.  Pass 2: one CTA per launch folds the
// partials in a fixed order (deterministic) into S_r, C_r and L.
// HBM-bound: each logits byte is read once.  The grids are one wave of
// resident CTAs.
//
// The gradient (the training step after the aggregation) has the global
// count C = sum_r C_r as its only denominator:
//   dL/dz_tv = (softmax(z_t)_v - [v == y_t]) / C   (counted tokens; else 0)
// The fused forward+backward counts the valid labels first (one CTA, labels
// only), then each token's warp computes the row's logsumexp exactly as the
// forward does, re-reads the row (now in L2) and writes dL/dz with 16-byte
// stores: logits read once from HBM, dlogits written once.
#include "common.cuh"
#include "prof.cuh"

namespace uly {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kLoadsInFlight = 8;
// The gradient pass keeps fewer loads in flight (its row comes from L2), so
// that the fused kernel fits three CTAs per SM like the partials kernel and
// both entry points share one grid.
constexpr int kGradLoads = 4;
constexpr float kLog2e = 1.4426950408889634f;

// 2^x on the special-function unit (flush-to-zero; x <= 0 here).
__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void merge(float &m, float &s, float m2, float s2) {
  // (m, s) represents sum exp(x - m) = s; combine two such pairs.
  const float mm = fmaxf(m, m2);
  if (mm == -INFINITY) return;
  s = s * exp2f((m - mm) * kLog2e) + s2 * exp2f((m2 - mm) * kLog2e);
  m = mm;
}

template <typename T>
__device__ __forceinline__ void load_vals(const uint4 &u, float (&x)[8]);

template <>
__device__ __forceinline__ void load_vals<__nv_bfloat16>(const uint4 &u, float (&x)[8]) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float2 f = __bfloat1622float2(h[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
}

// fp32 logits: one uint4 holds 4 values; pad the rest with -inf.
template <>
__device__ __forceinline__ void load_vals<float>(const uint4 &u, float (&x)[8]) {
  x[0] = __uint_as_float(u.x); x[1] = __uint_as_float(u.y);
  x[2] = __uint_as_float(u.z); x[3] = __uint_as_float(u.w);
  x[4] = x[5] = x[6] = x[7] = -INFINITY;
}

// Largest of the values one 16-byte vector holds (bf16: packed maxima).
template <typename T>
__device__ __forceinline__ float vec_max(const uint4 &u);

template <>
__device__ __forceinline__ float vec_max<__nv_bfloat16>(const uint4 &u) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
  const __nv_bfloat162 m = __hmax2(__hmax2(h[0], h[1]), __hmax2(h[2], h[3]));
  const float2 f = __bfloat1622float2(m);
  return fmaxf(f.x, f.y);
}

template <>
__device__ __forceinline__ float vec_max<float>(const uint4 &u) {
  return fmaxf(fmaxf(__uint_as_float(u.x), __uint_as_float(u.y)), fmaxf(__uint_as_float(u.z), __uint_as_float(u.w)));
}

// log sum_v exp(z_v) of one row, computed by the 32 lanes of a warp (every
// lane returns it).  STREAM: evict-first loads (the row is not read again).
template <typename T, bool STREAM>
__device__ __forceinline__ float row_lse(const T *rowp, int vocab, int lane) {
  constexpr int kPerVec = 16 / sizeof(T);
  const int vecs = vocab / kPerVec;  // vocab * sizeof(T) % 16 == 0 checked on the host
  const uint4 *row = reinterpret_cast<const uint4 *>(rowp);
  float m = -INFINITY, s = 0.f;
  for (int v0 = lane; v0 < vecs; v0 += 32 * kLoadsInFlight) {
    uint4 u[kLoadsInFlight];
#pragma unroll
    for (int k = 0; k < kLoadsInFlight; ++k) {
      const int v = v0 + k * 32;
      if (v < vecs) u[k] = STREAM ? __ldcs(row + v) : __ldg(row + v);
    }
    // one maximum (and at most one rescale) per group of loaded vectors
    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < kLoadsInFlight; ++k)
      if (v0 + k * 32 < vecs) mx = fmaxf(mx, vec_max<T>(u[k]));
    if (mx > m) {
      s = (m == -INFINITY) ? 0.f : s * exp2f((m - mx) * kLog2e);
      m = mx;
    }
    const float ml = (m == -INFINITY) ? 0.f : m * kLog2e;   // all -inf so far: every term is 0
    float s4[4] = {0.f, 0.f, 0.f, 0.f};   // four add chains, folded in a fixed order
#pragma unroll
    for (int k = 0; k < kLoadsInFlight; ++k) {
      if (v0 + k * 32 < vecs) {
        float x[8];
        load_vals<T>(u[k], x);
#pragma unroll
        for (int e = 0; e < 8; ++e) s4[e & 3] += ex2_mufu(fmaf(x[e], kLog2e, -ml));
      }
    }
    s += (s4[0] + s4[1]) + (s4[2] + s4[3]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, off);
    merge(m, s, m2, s2);
  }
  return m + logf(s);
}

// grid = (blocks_per_shard, P).  Partials: part_sum[r * nb + blockIdx.x], part_cnt[...].
template <typename T>
__global__ void __launch_bounds__(kThreads) ce_partial_kernel(
    const T *__restrict__ logits, const int32_t *__restrict__ labels, long long per_shard,
    int vocab, int ignore_index, double *__restrict__ part_sum, long long *__restrict__ part_cnt,
    int *err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y, nb = gridDim.x;
  double acc = 0.0;
  long long cnt = 0;
  for (long long tt = (long long)blockIdx.x * kWarps + warp; tt < per_shard;
       tt += (long long)nb * kWarps) {
    const long long t = (long long)r * per_shard + tt;
    const int y = __ldg(labels + t);
    if (y == ignore_index) continue;
    if (y < 0 || y >= vocab) {
      if (lane == 0) raise_error(err, ULY_ERR_LABEL);
      continue;
    }
    const float lse = row_lse<T, true>(logits + t * (long long)vocab, vocab, lane);
    if (lane == 0) {
      const float zy = static_cast<float>(logits[t * (long long)vocab + y]);
      acc += (double)lse - (double)zy;
      cnt += 1;
    }
  }
  __shared__ double sh_sum[kWarps];
  __shared__ long long sh_cnt[kWarps];
  if (lane == 0) { sh_sum[warp] = acc; sh_cnt[warp] = cnt; }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0;
    long long c = 0;
    for (int w = 0; w < kWarps; ++w) { a += sh_sum[w]; c += sh_cnt[w]; }  // fixed order
    part_sum[(long long)r * nb + blockIdx.x] = a;
    part_cnt[(long long)r * nb + blockIdx.x] = c;
  }
}

// Global count of valid labels (not the ignore index, inside [0, V)): one
// CTA, fixed-order reduction; written to *count.
__global__ void __launch_bounds__(1024) ce_count_kernel(const int32_t *__restrict__ labels, long long tokens,
                                                        int vocab, int ignore_index, long long *count) {
  long long c = 0;
  for (long long t = threadIdx.x; t < tokens; t += blockDim.x) {
    const int y = __ldg(labels + t);
    c += (y != ignore_index && y >= 0 && y < vocab) ? 1 : 0;
  }
  __shared__ long long sh[1024];
  sh[threadIdx.x] = c;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *count = sh[0];
}

template <typename T>
__device__ __forceinline__ uint4 pack_vals(const float (&x)[8]);
template <>
__device__ __forceinline__ uint4 pack_vals<__nv_bfloat16>(const float (&x)[8]) {
  uint4 u;
  uint32_t *w = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
    w[e] = *reinterpret_cast<uint32_t *>(&h);
  }
  return u;
}
template <>
__device__ __forceinline__ uint4 pack_vals<float>(const float (&x)[8]) {
  return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
}

// Loss partials as ce_partial_kernel, and dL/dz for every token of the shard.
template <typename T>
__global__ void __launch_bounds__(kThreads, 3) ce_fwd_bwd_kernel(
    const T *__restrict__ logits, const int32_t *__restrict__ labels, long long per_shard, int vocab,
    int ignore_index, const long long *__restrict__ count, T *__restrict__ dlogits,
    double *__restrict__ part_sum, long long *__restrict__ part_cnt, int *err) {
  constexpr int kPerVec = 16 / sizeof(T);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y, nb = gridDim.x;
  const int vecs = vocab / kPerVec;
  const long long C = *count;
  const float invC = C > 0 ? (float)(1.0 / (double)C) : 0.f;
  double acc = 0.0;
  long long cnt = 0;
  for (long long tt = (long long)blockIdx.x * kWarps + warp; tt < per_shard;
       tt += (long long)nb * kWarps) {
    const long long t = (long long)r * per_shard + tt;
    const int y = __ldg(labels + t);
    uint4 *drow = reinterpret_cast<uint4 *>(dlogits + t * (long long)vocab);
    const bool counted = y != ignore_index && y >= 0 && y < vocab;
    if (!counted) {
      if (y != ignore_index && lane == 0) raise_error(err, ULY_ERR_LABEL);
      for (int v = lane; v < vecs; v += 32) __stcs(drow + v, make_uint4(0, 0, 0, 0));
      continue;
    }
    const T *rowp = logits + t * (long long)vocab;
    const float lse = row_lse<T, false>(rowp, vocab, lane);
    if (lane == 0) {
      acc += (double)lse - (double)static_cast<float>(rowp[y]);
      cnt += 1;
    }
    // dL/dz = (exp(z - lse) - [v == y]) / C; the row is read again from L2,
    // four 16-byte loads in flight per lane
    const float lse2 = lse * kLog2e;
    const uint4 *row = reinterpret_cast<const uint4 *>(rowp);
    const int yv = y / kPerVec;
    for (int v0 = lane; v0 < vecs; v0 += 32 * kGradLoads) {
      uint4 u[kGradLoads];
#pragma unroll
      for (int k = 0; k < kGradLoads; ++k) {
        const int v = v0 + k * 32;
        if (v < vecs) u[k] = __ldg(row + v);
      }
#pragma unroll
      for (int k = 0; k < kGradLoads; ++k) {
        const int v = v0 + k * 32;
        if (v < vecs) {
          float x[8];
          load_vals<T>(u[k], x);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = ex2_mufu(fmaf(x[e], kLog2e, -lse2)) * invC;
          if (v == yv) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if (v * kPerVec + e == y) x[e] -= invC;
          }
          __stcs(drow + v, pack_vals<T>(x));
        }
      }
    }
  }
  __shared__ double sh_sum[kWarps];
  __shared__ long long sh_cnt[kWarps];
  if (lane == 0) { sh_sum[warp] = acc; sh_cnt[warp] = cnt; }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0;
    long long c = 0;
    for (int w = 0; w < kWarps; ++w) { a += sh_sum[w]; c += sh_cnt[w]; }  // fixed order
    part_sum[(long long)r * nb + blockIdx.x] = a;
    part_cnt[(long long)r * nb + blockIdx.x] = c;
  }
}

// One CTA: shard r's partials are folded by thread r in index order; then
// thread 0 folds the shards in rank order.
__global__ void __launch_bounds__(256) ce_finalize_kernel(
    const double *__restrict__ part_sum, const long long *__restrict__ part_cnt, int P, int nb,
    float *__restrict__ shard_sum, int64_t *__restrict__ shard_count, float *__restrict__ loss) {
  __shared__ double sh_s[256];
  __shared__ long long sh_c[256];
  for (int r = threadIdx.x; r < P; r += blockDim.x) {
    double a = 0.0;
    long long c = 0;
    for (int i = 0; i < nb; ++i) { a += part_sum[(long long)r * nb + i]; c += part_cnt[(long long)r * nb + i]; }
    shard_sum[r] = (float)a;
    shard_count[r] = c;
    if (r < 256) { sh_s[r] = a; sh_c[r] = c; }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0;
    long long c = 0;
    for (int r = 0; r < P; ++r) {
      if (r < 256) { a += sh_s[r]; c += sh_c[r]; }
      else { a += (double)shard_sum[r]; c += shard_count[r]; }
    }
    *loss = (float)(a / (double)c);  // 0/0 -> NaN when no token is valid
  }
}

// CTAs of `kernel` (kThreads threads, no dynamic shared memory) resident on
// the current device at once: its SMs times the occupancy (cached per device).
template <typename Kernel>
int resident_ctas(Kernel kernel) {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int sms = 0, per_sm = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) != cudaSuccess || sms <= 0 ||
      per_sm <= 0)
    return 148;
  const int n = sms * per_sm;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

}  // namespace

int loss_blocks_per_shard(int P, long long per_shard) {
  // the workspace bound: about four CTAs per SM in total, at most one warp per token
  long long nb = (4LL * 148 + P - 1) / P;
  long long need = (per_shard + kWarps - 1) / kWarps;
  if (nb > need) nb = need;
  if (nb < 1) nb = 1;
  return (int)nb;
}

// The CTAs of one launch: one wave of resident CTAs split over the P shards
// (each CTA's tokens are fixed by the grid stride, so a partial second wave
// would run on a fraction of the SMs), within the workspace bound.
static int launch_blocks_per_shard(int P, long long per_shard, int resident) {
  long long nb = resident / P;
  if (nb < 1) nb = 1;
  const int bound = loss_blocks_per_shard(P, per_shard);
  return (int)(nb < bound ? nb : bound);
}

// The grid of both loss entry points (the forward partials and the fused
// gradient): the same CTAs over the same tokens, so that their per-CTA
// partial sums, and so S_r, C_r and L, are equal bit for bit.  One wave of
// whichever of the two kernels has the lower occupancy.
static int loss_grid_blocks(int P, long long per_shard, int dtype) {
  const int a = dtype == ULY_BF16 ? resident_ctas(ce_partial_kernel<__nv_bfloat16>)
                                  : resident_ctas(ce_partial_kernel<float>);
  const int b = dtype == ULY_BF16 ? resident_ctas(ce_fwd_bwd_kernel<__nv_bfloat16>)
                                  : resident_ctas(ce_fwd_bwd_kernel<float>);
  return launch_blocks_per_shard(P, per_shard, a < b ? a : b);
}

size_t loss_workspace_bytes(int P, long long per_shard) {
  const size_t nb = (size_t)loss_blocks_per_shard(P, per_shard);
  return nb * (size_t)P * (sizeof(double) + sizeof(long long));
}

uly_status loss_validate(int32_t P, int64_t tokens, int32_t vocab, int32_t dtype, const void *logits,
                         const int32_t *labels, const float *shard_sum, const int64_t *shard_count,
                         const float *loss) {
  if (!logits || !labels || !shard_sum || !shard_count || !loss) return ULY_ERR_NULL;
  if (dtype != ULY_BF16 && dtype != ULY_F32) return ULY_ERR_DTYPE;
  if (P <= 0 || P > 65535 || tokens < 0 || vocab <= 0) return ULY_ERR_SHAPE;
  if (tokens % P) return ULY_ERR_SHAPE;
  const int eb = dtype == ULY_BF16 ? 2 : 4;
  if (((long long)vocab * eb) % 16) return ULY_ERR_ALIGN;
  if (!aligned16(logits) || !aligned16(labels)) return ULY_ERR_ALIGN;
  return ULY_OK;
}

// `ws` holds nb*P doubles followed by nb*P long longs.
uly_status loss_launch(int32_t P, int64_t tokens, int32_t vocab, int32_t dtype, const void *logits,
                       const int32_t *labels, int32_t ignore_index, float *shard_sum,
                       int64_t *shard_count, float *loss, void *ws, cudaStream_t stream) {
  const long long per = tokens / P;
  const int nb_ws = loss_blocks_per_shard(P, per);   // the workspace layout
  const int nb = loss_grid_blocks(P, per, dtype);
  double *psum = static_cast<double *>(ws);
  long long *pcnt = reinterpret_cast<long long *>(psum + (size_t)nb_ws * P);
  dim3 grid(nb, P);
  prof::Scope s1(prof::K_LOSS_PARTIAL, stream);
  if (dtype == ULY_BF16)
    ce_partial_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(logits), labels, per, vocab, ignore_index, psum, pcnt,
        error_word());
  else
    ce_partial_kernel<float><<<grid, kThreads, 0, stream>>>(
        static_cast<const float *>(logits), labels, per, vocab, ignore_index, psum, pcnt,
        error_word());
  s1.end();
  prof::Scope s2(prof::K_LOSS_FINALIZE, stream);
  ce_finalize_kernel<<<1, 256, 0, stream>>>(psum, pcnt, P, nb, shard_sum, shard_count, loss);
  note_launches(2);
  return last_launch_status();
}

// Fused forward + backward.  `ws`: the forward's partials followed by one
// long long (the global count of valid labels).
size_t loss_bwd_workspace_bytes(int P, long long per_shard) {
  return ((loss_workspace_bytes(P, per_shard) + 15) & ~size_t(15)) + 16;
}

uly_status loss_bwd_launch(int32_t P, int64_t tokens, int32_t vocab, int32_t dtype, const void *logits,
                           const int32_t *labels, int32_t ignore_index, void *dlogits, float *shard_sum,
                           int64_t *shard_count, float *loss, void *ws, cudaStream_t stream) {
  const long long per = tokens / P;
  const int nb_ws = loss_blocks_per_shard(P, per);   // the workspace layout
  const int nb = loss_grid_blocks(P, per, dtype);
  double *psum = static_cast<double *>(ws);
  long long *pcnt = reinterpret_cast<long long *>(psum + (size_t)nb_ws * P);
  long long *count = reinterpret_cast<long long *>(static_cast<char *>(ws) +
                                                   ((loss_workspace_bytes(P, per) + 15) & ~size_t(15)));
  dim3 grid(nb, P);
  prof::Scope s1(prof::K_LOSS_FWD_BWD, stream);
  ce_count_kernel<<<1, 1024, 0, stream>>>(labels, tokens, vocab, ignore_index, count);
  if (dtype == ULY_BF16)
    ce_fwd_bwd_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(logits), labels, per, vocab, ignore_index, count,
        static_cast<__nv_bfloat16 *>(dlogits), psum, pcnt, error_word());
  else
    ce_fwd_bwd_kernel<float><<<grid, kThreads, 0, stream>>>(
        static_cast<const float *>(logits), labels, per, vocab, ignore_index, count,
        static_cast<float *>(dlogits), psum, pcnt, error_word());
  s1.end();
  prof::Scope s2(prof::K_LOSS_FINALIZE, stream);
  ce_finalize_kernel<<<1, 256, 0, stream>>>(psum, pcnt, P, nb, shard_sum, shard_count, loss);
  note_launches(3);
  return last_launch_status();
}

}  // namespace uly
