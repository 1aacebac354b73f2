// The projections either side of Ulysses attention, on the 5th-generation
// tensor cores ("Paralelismul de Secvență Ulysses", section "Mecanismul de
// funcționare Ulysses", steps 2-3 and 5-6):
//
//  QKV: every rank projects its own tokens, [Q K V] = X W^T, rotates Q and K by
//  each token's position in the whole sequence (rank r's local token tt sits at
//  t = r*n/P + tt; the ms-swift page, section 6.2, lists a RoPE that ignores the
//  shard's offset as a failure), and the first all-to-all is folded into the
//  epilogue: every output row is written straight to its place in the head
//  layout, so the projected Q/K/V never exist in the seq layout.
//
//  O-proj: the second all-to-all is folded into the operand load: a CTA's A
//  tile (128 positions x 64 features of one head) is read by TMA directly from
//  the head layout, and Y = O W_o^T is written in the seq layout.
//
// Both are C[M][N] = A[M][K] B[N][K]^T with bf16 operands and fp32
// accumulation, tiles of 128 x 256 (two heads of 128 columns for QKV), K in
// 64-column steps (one 128-byte swizzle span).  The kernel is persistent:
// one CTA per SM walks the tiles (N fastest, so CTAs running at the same time
// share their A rows in L2).
//
// Warp roles (192 threads):
//   warp 0     TMA producer: A and B k-steps into a 4-stage ring (48 KB each)
//   warp 1     TMEM allocator and MMA issuer: 4 MMAs (M=128 N=256 K=16) per
//              stage into one of two 256-column accumulators
//   warps 2-5  epilogue: one thread per accumulator row (TMEM lane) reads its
//              row, applies the rotation (QKV), rounds to bf16 and stores;
//              the other accumulator is filled by the next tile meanwhile.
// Every wait is bounded (ULY_ERR_TIMEOUT); nothing can spin forever.
#include <atomic>

#include "prof.cuh"
#include "sm100.cuh"

namespace uly {

using namespace sm100;

bool make_tmap_heads_bf16(CUtensorMap *map, const void *base, int d, int n, int heads, int box_rows);

namespace {

// 2-D tiled load into shared memory, completion counted on `bar` (bytes).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0,
                                            int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

// 2-D bf16 map over a row-major [rows][inner] matrix with box_inner x
// box_rows boxes (box_inner * 2 = 128 bytes: one 128-byte swizzle span);
// elements past either edge read as zero.
bool make_tmap_rows_bf16(CUtensorMap *map, const void *base, long long inner, long long rows, int box_inner,
                         int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!enc) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                   es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr int kBM = 128, kBN = 256, kBK = 64, kHD = 128;
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr uint32_t kABytes = kBM * kBK * 2;             // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;             // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;     // 48 KB
constexpr uint32_t kOffBar = kStages * kStageBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;   // barriers + alignment slack
constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(kBM, kBN, false, false);
constexpr uint32_t kIdescKM = sm100::idesc_bf16_f32(kBM, kBN, false, true);   // B MN-major
constexpr uint32_t kIdescMK = sm100::idesc_bf16_f32(kBM, kBN, true, false);   // A MN-major
constexpr uint32_t kIdescMM = sm100::idesc_bf16_f32(kBM, kBN, true, true);

// QKV / OPROJ: the forward projections.  The backward ones (the adjoints of
// steps 2-3 and 5-6) reuse the same pipeline with other operand layouts and
// epilogues:
//   DX:    dX[M][hidden]  = dY[M][Nqkv] W[Nqkv][hidden]      A K-major, B MN-major, bf16 rows
//   DW:    dW[Nqkv][hidden] = dY^T X  (sum over all tokens)   A, B MN-major, fp32 rows
//   DO:    dO = dY_o[M][hidden] W_o[hidden][H*d] -> head layout  A K-major, B MN-major
//   DWO:   dW_o[hidden][H*d] = dY_o^T O_seq                   A, B MN-major, fp32 rows
// An MN-major operand (its M or N index contiguous in memory, K along rows)
// arrives as 64-row TMA boxes of 64 contiguous elements, one per 64 columns
// of the tile: the same 16 KB (A) and 32 KB (B) per stage.
enum Mode { MODE_QKV = 0, MODE_OPROJ = 1, MODE_DX = 2, MODE_DW = 3, MODE_DO = 4, MODE_DWO = 5 };

struct ProjParams {
  int mode;
  int K;             // reduction length (hidden for QKV, H*d for the output projection)
  int m_tiles, n_tiles;
  int B, n, s, P;
  int hl, gl, H, G;  // query / KV heads per rank and in total
  long long M;       // QKV: rows of X (P*B*s)
  int hidden;        // output projection: width of Y
  int tiles_per_b;   // output projection: position tiles per batch row
  const float4 *rope;        // [max_pos][32] float4 = (cos e, sin e, cos e+1, sin e+1)
  int max_pos;
  const int32_t *positions;  // nullable [B][n]
  __nv_bfloat16 *q, *k, *v;  // QKV outputs, head layout
  __nv_bfloat16 *y;          // output projection result, seq layout
  int a_mn, b_mn;            // operand A / B is MN-major (2-D map with 64 x 64 boxes)
  long long ldc;             // DX / DW / DWO: row stride of C in elements
  __nv_bfloat16 *c16;        // DX: bf16 C
  float *c32;                // DW / DWO: fp32 C
  long long M_rows;          // DX / DW / DWO: rows of C (rows past it are not stored)
  int ksplit;                // DW / DWO: 1, or 2 = each tile's k-steps in two halves (work units),
                             // added into a zeroed C with fp32 reduce-adds
  int *err;
  long long wait_limit;      // cycles a pipeline wait may last (wait_limit_cycles())
};

__device__ __forceinline__ void store_row_chunk(__nv_bfloat16 *dst, const float (&x)[32]) {
  uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint4 w;
    w.x = pack_bf16x2(x[8 * u + 0], x[8 * u + 1]);
    w.y = pack_bf16x2(x[8 * u + 2], x[8 * u + 3]);
    w.z = pack_bf16x2(x[8 * u + 4], x[8 * u + 5]);
    w.w = pack_bf16x2(x[8 * u + 6], x[8 * u + 7]);
    d4[u] = w;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    proj_sm100_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const ProjParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  enum { B_FULL = 0, B_EMPTY = kStages, B_ACCF = 2 * kStages, B_ACCE = B_ACCF + 2, B_DRAIN = B_ACCE + 2,
         B_N = B_DRAIN + 1 };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffBar + 8 * B_N);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffBar + 8 * B_N + 4);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = prm.m_tiles * prm.n_tiles;
  const int KT = (prm.K + kBK - 1) / kBK;   // a ragged last k-step reads zeros past K
  const int ks = prm.ksplit;                // work unit u: tile u / ks, k-steps of its part u % ks
  const int nunits = ntiles * ks;

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_N; ++i) mbar_init(bar(i), (i == B_ACCE || i == B_ACCE + 1) ? 128 : 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      long long idx = 0;   // k-steps issued so far (ring position)
      bool ok = true;
      for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
        const int tile = u / ks, sp = u - tile * ks;
        const int kt0 = (int)((long long)KT * sp / ks), kt1 = (int)((long long)KT * (sp + 1) / ks);
        const int mt = tile / prm.n_tiles, nt = tile - mt * prm.n_tiles;
        const int n0 = nt * kBN;
        int b = 0, t0 = 0;
        if (prm.mode == MODE_OPROJ) {
          b = mt / prm.tiles_per_b;
          t0 = (mt - b * prm.tiles_per_b) * kBM;
        }
        for (int kt = kt0; kt < kt1; ++kt, ++idx) {
          const int stage = (int)(idx % kStages);
          const long long use = idx / kStages;
          if (use > 0 && !mbar_wait(bar(B_EMPTY + stage), (uint32_t)((use - 1) & 1), abort_flag, prm.err, prm.wait_limit)) {
            ok = false;
            break;
          }
          const uint32_t sA = sb + stage * kStageBytes, sB = sA + kABytes;
          mbar_arrive_expect_tx(bar(B_FULL + stage), kStageBytes);
          if (prm.mode == MODE_OPROJ) {
            // k-step kt covers features [64 (kt % 2), +64) of query head kt / 2,
            // held by rank kt / 2 / hl as its local head (kt / 2) % hl
            const int qh = kt >> 1, r2 = qh / prm.hl, hh = qh - r2 * prm.hl;
            tma_load_3d(sA, &tmA, bar(B_FULL + stage), (kt & 1) * kBK, t0, (r2 * prm.B + b) * prm.hl + hh);
          } else if (prm.a_mn) {
            for (int c = 0; c < kBM / 64; ++c)
              tma_load_2d(sA + c * 8192, &tmA, bar(B_FULL + stage), mt * kBM + 64 * c, kt * kBK);
          } else {
            tma_load_2d(sA, &tmA, bar(B_FULL + stage), kt * kBK, mt * kBM);
          }
          if (prm.b_mn) {
            for (int c = 0; c < kBN / 64; ++c)
              tma_load_2d(sB + c * 8192, &tmB, bar(B_FULL + stage), n0 + 64 * c, kt * kBK);
          } else {
            tma_load_2d(sB, &tmB, bar(B_FULL + stage), kt * kBK, n0);
          }
        }
      }
      // every copy issued lands before the CTA can exit, also when the MMA
      // thread gave up waiting for it; on the normal path these return at once
      for (long long j = (idx > kStages ? idx - kStages : 0); j < idx; ++j)
        mbar_wait(bar(B_FULL + (int)(j % kStages)), (uint32_t)((j / kStages) & 1), nullptr, prm.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      long long idx = 0;
      bool ok = true;
      int it = 0;
      for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x, ++it) {
        const int sp = u % ks;
        const int kt0 = (int)((long long)KT * sp / ks), kt1 = (int)((long long)KT * (sp + 1) / ks);
        const int buf = it & 1;
        if (it >= 2) {
          ok = mbar_wait(bar(B_ACCE + buf), (uint32_t)(((it >> 1) - 1) & 1), abort_flag, prm.err, prm.wait_limit);
          if (!ok) break;
          tc_fence_after();
        }
        const uint32_t acc = tmem + buf * kBN;
        for (int kt = kt0; kt < kt1; ++kt, ++idx) {
          const int stage = (int)(idx % kStages);
          const uint32_t sA = sb + stage * kStageBytes, sB = sA + kABytes;
          // K-major: 16 K-elements are 32 bytes along a row; MN-major: 16 K-rows
          // are 2048 bytes, the 64-element MN chunks 8 KB apart (LBO)
          const uint64_t da = prm.a_mn ? sdesc_sw128(sA, 8192, 1024) : sdesc_sw128(sA, 16, 1024);
          const uint64_t db = prm.b_mn ? sdesc_sw128(sB, 8192, 1024) : sdesc_sw128(sB, 16, 1024);
          const uint32_t astep = prm.a_mn ? 2048 : 32, bstep = prm.b_mn ? 2048 : 32;
          const uint32_t idesc = prm.a_mn ? (prm.b_mn ? kIdescMM : kIdescMK) : (prm.b_mn ? kIdescKM : kIdesc);
          ok = mbar_wait(bar(B_FULL + stage), (uint32_t)((idx / kStages) & 1), abort_flag, prm.err, prm.wait_limit);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16_ss(acc, sdesc_add(da, kk * astep), sdesc_add(db, kk * bstep), idesc,
                        (kt > kt0 || kk > 0) ? 1u : 0u);
          tc_commit(bar(B_EMPTY + stage));
        }
        if (!ok) break;
        tc_commit(bar(B_ACCF + buf));
      }
      // drain: every MMA issued has completed before TMEM can be released
      tc_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, nullptr, prm.err);
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    int it = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
      const int tile = u / ks;
      const int buf = it & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_ACCF + buf), (uint32_t)((it >> 1) & 1), abort_flag, prm.err, prm.wait_limit)))
        break;
      tc_fence_after();
      const int mt = tile / prm.n_tiles, nt = tile - mt * prm.n_tiles;
      const uint32_t acc = tmem + lane_off + buf * kBN;
      if (prm.mode == MODE_DX || prm.mode == MODE_DW || prm.mode == MODE_DWO) {
        // plain row-major C: bf16 (dX) or fp32 (the weight gradients)
        const long long m = (long long)mt * kBM + row;
        const bool valid = m < prm.M_rows;
        const long long c0 = m * prm.ldc + (long long)nt * kBN;
#pragma unroll 1
        for (int c = 0; c < kBN; c += 32) {
          uint32_t a[32];
          tmem_ld32(acc + c, a);
          if (valid) {
            if (prm.mode == MODE_DX) {
              float x[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(a[e]);
              store_row_chunk(prm.c16 + c0 + c, x);
            } else if (ks == 1) {
              float4 *d4 = reinterpret_cast<float4 *>(prm.c32 + c0 + c);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                d4[q] = make_float4(__uint_as_float(a[4 * q]), __uint_as_float(a[4 * q + 1]),
                                    __uint_as_float(a[4 * q + 2]), __uint_as_float(a[4 * q + 3]));
            } else {
              // the tile's two halves meet in L2; with two partials added
              // into zero, either order gives the same bits
              float4 *d4 = reinterpret_cast<float4 *>(prm.c32 + c0 + c);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                atomicAdd(d4 + q, make_float4(__uint_as_float(a[4 * q]), __uint_as_float(a[4 * q + 1]),
                                              __uint_as_float(a[4 * q + 2]), __uint_as_float(a[4 * q + 3])));
            }
          }
        }
      } else if (prm.mode == MODE_QKV || prm.mode == MODE_DO) {
        const long long m = (long long)mt * kBM + row;
        const bool valid = m < prm.M;
        int b = 0, t = 0, pos = 0;
        if (valid) {
          const long long bs = (long long)prm.B * prm.s;
          const int r = (int)(m / bs);
          const long long rem = m - (long long)r * bs;
          b = (int)(rem / prm.s);
          const int tt = (int)(rem - (long long)b * prm.s);
          t = r * prm.s + tt;
          if (prm.mode == MODE_QKV) {
            pos = prm.positions ? __ldg(prm.positions + (long long)b * prm.n + t) : t;
            if (pos < 0 || pos >= prm.max_pos) {
              raise_error(prm.err, ULY_ERR_SHAPE);
              pos = 0;
            }
          }
        }
#pragma unroll 1
        for (int hs = 0; hs < 2; ++hs) {
          const int j = nt * 2 + hs;         // output head: H query, G key, G value heads
          __nv_bfloat16 *base;
          int heads_local, jj;
          // QKV: H query, G key, G value heads (Q and K rotated); DO: the H
          // query heads of dO, not rotated
          if (j < prm.H) { base = prm.q; heads_local = prm.hl; jj = j; }
          else if (j < prm.H + prm.G) { base = prm.k; heads_local = prm.gl; jj = j - prm.H; }
          else { base = prm.v; heads_local = prm.gl; jj = j - prm.H - prm.G; }
          const bool rot = prm.mode == MODE_QKV && j < prm.H + prm.G;
          const int r2 = jj / heads_local, hh = jj - r2 * heads_local;
          __nv_bfloat16 *dst = base + ((((long long)r2 * prm.B + b) * heads_local + hh) * prm.n + t) * kHD;
#pragma unroll 1
          for (int c0 = 0; c0 < kHD / 2; c0 += 32) {
            uint32_t a1[32], a2[32];
            tmem_ld32(acc + hs * kHD + c0, a1);
            tmem_ld32(acc + hs * kHD + kHD / 2 + c0, a2);
            float y1[32], y2[32];
            if (rot) {
              const float4 *cs = prm.rope + (long long)pos * (kHD / 4) + c0 / 2;
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float4 w = __ldg(cs + e / 2);
                const float x1a = __uint_as_float(a1[e]), x2a = __uint_as_float(a2[e]);
                const float x1b = __uint_as_float(a1[e + 1]), x2b = __uint_as_float(a2[e + 1]);
                y1[e] = x1a * w.x - x2a * w.y;
                y2[e] = x2a * w.x + x1a * w.y;
                y1[e + 1] = x1b * w.z - x2b * w.w;
                y2[e + 1] = x2b * w.z + x1b * w.w;
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                y1[e] = __uint_as_float(a1[e]);
                y2[e] = __uint_as_float(a2[e]);
              }
            }
            if (valid) {
              store_row_chunk(dst + c0, y1);
              store_row_chunk(dst + kHD / 2 + c0, y2);
            }
          }
        }
      } else {
        const int b = mt / prm.tiles_per_b;
        const int t = (mt - b * prm.tiles_per_b) * kBM + row;
        const bool valid = t < prm.n;
        const int r = valid ? t / prm.s : 0, tt = valid ? t - r * prm.s : 0;
        __nv_bfloat16 *dst = prm.y + (((long long)r * prm.B + b) * prm.s + tt) * prm.hidden + nt * kBN;
#pragma unroll 1
        for (int c = 0; c < kBN; c += 32) {
          uint32_t a[32];
          tmem_ld32(acc + c, a);
          float x[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(a[e]);
          if (valid) store_row_chunk(dst + c, x);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_ACCE + buf));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// cos / sin of position p times base^(-2e/d), computed in double and rounded
// once to float; laid out [p][e/2] as float4 (cos e, sin e, cos e+1, sin e+1).
__global__ void rope_table_kernel(int max_pos, int half, double base, float *table) {
  const long long total = (long long)max_pos * half;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int p = (int)(i / half), e = (int)(i - (long long)p * half);
    const double theta = pow(base, -2.0 * e / (2.0 * half));
    double sn, cs;
    sincos((double)p * theta, &sn, &cs);
    table[2 * i] = (float)cs;
    table[2 * i + 1] = (float)sn;
  }
}

// dY of the QKV projection's backward, seq layout [M][(H + 2G) * 128] with
// M = P*B*s tokens (m = (r*B + b)*s + tt, position t = r*s + tt): output head
// j's gradient row comes from the head layout (the inverse of the folded
// all-to-all) and, for query and key heads, is rotated back by -pos (the
// transpose of the rotation: d1 = g1 cos + g2 sin, d2 = g2 cos - g1 sin for
// the pair (e, e + 64)).  8 threads per row, 8 pairs each; HBM-bound.
__global__ void __launch_bounds__(512) qkv_dy_kernel(const __nv_bfloat16 *__restrict__ dq,
                                                      const __nv_bfloat16 *__restrict__ dk,
                                                      const __nv_bfloat16 *__restrict__ dv,
                                                      const float4 *__restrict__ rope, int max_pos,
                                                      const int32_t *__restrict__ positions,
                                                      __nv_bfloat16 *__restrict__ dy, int B, int n, int s, int H,
                                                      int G, int hl, int gl, long long M, int *err) {
  // eight threads per output row (one head of one token): thread l moves the
  // elements [8l, 8l + 8) and [64 + 8l, 64 + 8l + 8) as 16-byte vectors, so it
  // holds the rotary pairs (e, e + 64) it rotates.  Two tokens per iteration,
  // all their loads issued before any arithmetic.
  constexpr int kTok = 2;
  const int l = threadIdx.x & 7, grp = threadIdx.x >> 3, ngrp = blockDim.x >> 3;
  const int J = H + 2 * G;
  const long long bs = (long long)B * s;
  for (long long m0 = (long long)blockIdx.x * kTok; m0 < M; m0 += (long long)gridDim.x * kTok) {
    int b_[kTok], t_[kTok];
    float4 w[kTok][4];   // cos / sin of this thread's eight pairs (two per float4)
#pragma unroll
    for (int k = 0; k < kTok; ++k) {
      const long long m = m0 + k < M ? m0 + k : m0;   // a past-the-end token repeats m0 (not stored)
      const int r = (int)(m / bs);
      const long long rem = m - (long long)r * bs;
      b_[k] = (int)(rem / s);
      t_[k] = r * s + (int)(rem - (long long)b_[k] * s);
      int pos = positions ? __ldg(positions + (long long)b_[k] * n + t_[k]) : t_[k];
      if (pos < 0 || pos >= max_pos) {
        if (threadIdx.x == 0) raise_error(err, ULY_ERR_SHAPE);
        pos = 0;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) w[k][q] = __ldg(rope + (long long)pos * (kHD / 4) + 4 * l + q);
    }
    for (int j = grp; j < J; j += ngrp) {
      const __nv_bfloat16 *base;
      int heads_local, jj;
      if (j < H) { base = dq; heads_local = hl; jj = j; }
      else if (j < H + G) { base = dk; heads_local = gl; jj = j - H; }
      else { base = dv; heads_local = gl; jj = j - H - G; }
      const int r2 = jj / heads_local, hh = jj - r2 * heads_local;
      uint4 a[kTok], c[kTok];
#pragma unroll
      for (int k = 0; k < kTok; ++k) {
        const __nv_bfloat16 *src = base + ((((long long)r2 * B + b_[k]) * heads_local + hh) * n + t_[k]) * kHD;
        a[k] = __ldg(reinterpret_cast<const uint4 *>(src) + l);        // elements 8l .. 8l+7
        c[k] = __ldg(reinterpret_cast<const uint4 *>(src + 64) + l);   // elements 64+8l ..
      }
#pragma unroll
      for (int k = 0; k < kTok; ++k) {
        if (m0 + k >= M) break;
        uint4 o1 = a[k], o2 = c[k];
        if (j < H + G) {
          const uint32_t av[4] = {a[k].x, a[k].y, a[k].z, a[k].w}, cv[4] = {c[k].x, c[k].y, c[k].z, c[k].w};
          uint32_t p1[4], p2[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {   // elements 8l + 2q, 8l + 2q + 1 and their partners + 64
            const float2 g1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&av[q]));
            const float2 g2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&cv[q]));
            const float4 wq = w[k][q];
            p1[q] = pack_bf16x2(g1.x * wq.x + g2.x * wq.y, g1.y * wq.z + g2.y * wq.w);
            p2[q] = pack_bf16x2(g2.x * wq.x - g1.x * wq.y, g2.y * wq.z - g1.y * wq.w);
          }
          o1 = make_uint4(p1[0], p1[1], p1[2], p1[3]);
          o2 = make_uint4(p2[0], p2[1], p2[2], p2[3]);
        }
        __nv_bfloat16 *out = dy + ((m0 + k) * J + j) * (long long)kHD;
        reinterpret_cast<uint4 *>(out)[l] = o1;
        reinterpret_cast<uint4 *>(out + 64)[l] = o2;
      }
    }
  }
}

uly_status launch_proj(const CUtensorMap &ta, const CUtensorMap &tb, const ProjParams &prm_in, int kernel_id,
                       cudaStream_t stream) {
  ProjParams prm = prm_in;
  prm.ksplit = 1;
  // the shared-memory opt-in is a per-device attribute: set it once on every
  // device this process launches on
  static std::atomic<uint64_t> attr_devices{0};
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return ULY_ERR_CUDA;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (!bit || !(attr_devices.load(std::memory_order_acquire) & bit)) {
    if (cudaFuncSetAttribute(proj_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
        cudaSuccess)
      return ULY_ERR_CUDA;
    attr_devices.fetch_or(bit, std::memory_order_acq_rel);
  }
  // The weight gradients contract over every token (long k loops) into few
  // output tiles: when halving each tile's k-steps fills the last wave of the
  // persistent grid better, a work unit is half a tile, added into a zeroed C.
  const int ntiles = prm.m_tiles * prm.n_tiles;
  if ((prm.mode == MODE_DW || prm.mode == MODE_DWO) && (prm.K + kBK - 1) / kBK >= 64) {
    auto fill = [&](int units) { return (double)units / ((double)((units + sms - 1) / sms) * sms); };
    if (fill(2 * ntiles) > fill(ntiles) + 0.02) prm.ksplit = 2;
  }
  const int nunits = ntiles * prm.ksplit;
  const int grid = nunits < sms ? nunits : sms;
  prof::Scope scope(kernel_id, stream);   // the zeroing of C is part of the timed entry point
  if (prm.ksplit == 2 &&
      cudaMemsetAsync(prm.c32, 0, (size_t)prm.M_rows * (size_t)prm.ldc * sizeof(float), stream) != cudaSuccess)
    return ULY_ERR_CUDA;
  proj_sm100_kernel<<<grid, kThreads, kSmemBytes, stream>>>(ta, tb, prm);
  note_launches(1);
  return last_launch_status();
}

}  // namespace

uly_status rope_table_launch(int32_t max_pos, int32_t head_dim, double base, float *table, cudaStream_t stream) {
  const long long total = (long long)max_pos * (head_dim / 2);
  long long blocks = (total + 255) / 256;
  if (blocks > 148LL * 32) blocks = 148LL * 32;
  prof::Scope scope(prof::K_ROPE_TABLE, stream);
  rope_table_kernel<<<(unsigned)blocks, 256, 0, stream>>>(max_pos, head_dim / 2, base, table);
  note_launches(1);
  return last_launch_status();
}

uly_status qkv_proj_launch(int32_t B, int32_t n, int32_t P, int32_t hidden, int32_t H, int32_t G,
                           const void *x, const void *w, const float *rope, int32_t max_pos,
                           const int32_t *positions, void *q, void *k, void *v, cudaStream_t stream) {
  const long long M = (long long)B * n;
  const long long N = (long long)(H + 2 * G) * kHD;
  CUtensorMap ta, tb;
  if (!make_tmap_rows_bf16(&ta, x, hidden, M, kBK, kBM) || !make_tmap_rows_bf16(&tb, w, hidden, N, kBK, kBN))
    return ULY_ERR_CUDA;
  ProjParams prm = {};
  prm.mode = MODE_QKV;
  prm.K = hidden;
  prm.m_tiles = (int)((M + kBM - 1) / kBM);
  prm.n_tiles = (int)(N / kBN);
  prm.B = B; prm.n = n; prm.s = n / P; prm.P = P;
  prm.H = H; prm.G = G; prm.hl = H / P; prm.gl = G / P;
  prm.M = M;
  prm.rope = reinterpret_cast<const float4 *>(rope);
  prm.max_pos = max_pos;
  prm.positions = positions;
  prm.q = static_cast<__nv_bfloat16 *>(q);
  prm.k = static_cast<__nv_bfloat16 *>(k);
  prm.v = static_cast<__nv_bfloat16 *>(v);
  prm.err = error_word();
  prm.wait_limit = wait_limit_cycles();
  return launch_proj(ta, tb, prm, prof::K_QKV_PROJ, stream);
}

// Backward of the QKV projection: dY pre-pass into `dy` (workspace), then
// dX = dY W and dW = dY^T X on the tensor cores.
uly_status qkv_proj_bwd_launch(int32_t B, int32_t n, int32_t P, int32_t hidden, int32_t H, int32_t G,
                               const void *x, const void *w, const float *rope, int32_t max_pos,
                               const int32_t *positions, const void *dq, const void *dk, const void *dv, void *dx,
                               float *dw, void *dy, cudaStream_t stream) {
  const long long M = (long long)B * n;
  const long long N = (long long)(H + 2 * G) * kHD;
  {
    // eight threads per head of a token: one token per CTA iteration
    const int J = H + 2 * G;
    int threads = ((8 * J + 31) / 32) * 32;
    if (threads > 512) threads = 512;   // more heads: a group takes several rows of a token
    // one wave of resident CTAs (each CTA's tokens are fixed by the grid stride)
    int per_sm = 0, dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, qkv_dy_kernel, threads, 0) != cudaSuccess || per_sm < 1)
      return ULY_ERR_CUDA;
    long long blocks = (long long)sms * per_sm;
    if (blocks > (M + 1) / 2) blocks = (M + 1) / 2;
    if (blocks < 1) blocks = 1;
    prof::Scope scope(prof::K_QKV_DY, stream);
    qkv_dy_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(dq), static_cast<const __nv_bfloat16 *>(dk),
        static_cast<const __nv_bfloat16 *>(dv), reinterpret_cast<const float4 *>(rope), max_pos, positions,
        static_cast<__nv_bfloat16 *>(dy), B, n, n / P, H, G, H / P, G / P, M, error_word());
    note_launches(1);
    if (last_launch_status() != ULY_OK) return ULY_ERR_CUDA;
  }
  CUtensorMap ta, tb;
  ProjParams prm = {};
  prm.B = B; prm.n = n; prm.s = n / P; prm.P = P;
  prm.err = error_word();
  prm.wait_limit = wait_limit_cycles();
  // dX[M][hidden] = dY[M][N] W[N][hidden]
  if (!make_tmap_rows_bf16(&ta, dy, N, M, kBK, kBM) || !make_tmap_rows_bf16(&tb, w, hidden, N, 64, 64))
    return ULY_ERR_CUDA;
  prm.mode = MODE_DX;
  prm.K = (int)N;
  prm.m_tiles = (int)((M + kBM - 1) / kBM);
  prm.n_tiles = hidden / kBN;
  prm.a_mn = 0;
  prm.b_mn = 1;
  prm.ldc = hidden;
  prm.M_rows = M;
  prm.c16 = static_cast<__nv_bfloat16 *>(dx);
  uly_status st = launch_proj(ta, tb, prm, prof::K_QKV_DX, stream);
  if (st != ULY_OK) return st;
  // dW[N][hidden] = dY^T X, summed over every token
  if (!make_tmap_rows_bf16(&ta, dy, N, M, 64, 64) || !make_tmap_rows_bf16(&tb, x, hidden, M, 64, 64))
    return ULY_ERR_CUDA;
  prm.mode = MODE_DW;
  prm.K = (int)M;
  prm.m_tiles = (int)(N / kBM);
  prm.n_tiles = hidden / kBN;
  prm.a_mn = 1;
  prm.b_mn = 1;
  prm.ldc = hidden;
  prm.M_rows = N;
  prm.c16 = nullptr;
  prm.c32 = dw;
  return launch_proj(ta, tb, prm, prof::K_QKV_DW, stream);
}

// Backward of the output projection: dO = dY W_o stored in the head layout
// (the first all-to-all in the epilogue), dW_o = dY^T O with O in the seq layout.
uly_status o_proj_bwd_launch(int32_t B, int32_t n, int32_t P, int32_t hidden, int32_t H, const void *o_seq,
                             const void *w_o, const void *dy, void *do_head, float *dw_o, cudaStream_t stream) {
  const long long M = (long long)B * n;
  const long long HD = (long long)H * kHD;
  CUtensorMap ta, tb;
  ProjParams prm = {};
  prm.B = B; prm.n = n; prm.s = n / P; prm.P = P;
  prm.H = H; prm.G = 0; prm.hl = H / P; prm.gl = 1;
  prm.M = M;
  prm.err = error_word();
  prm.wait_limit = wait_limit_cycles();
  if (!make_tmap_rows_bf16(&ta, dy, hidden, M, kBK, kBM) || !make_tmap_rows_bf16(&tb, w_o, HD, hidden, 64, 64))
    return ULY_ERR_CUDA;
  prm.mode = MODE_DO;
  prm.K = hidden;
  prm.m_tiles = (int)((M + kBM - 1) / kBM);
  prm.n_tiles = (int)(HD / kBN);
  prm.a_mn = 0;
  prm.b_mn = 1;
  prm.q = static_cast<__nv_bfloat16 *>(do_head);
  uly_status st = launch_proj(ta, tb, prm, prof::K_O_PROJ_DO, stream);
  if (st != ULY_OK) return st;
  if (!make_tmap_rows_bf16(&ta, dy, hidden, M, 64, 64) || !make_tmap_rows_bf16(&tb, o_seq, HD, M, 64, 64))
    return ULY_ERR_CUDA;
  prm.mode = MODE_DWO;
  prm.K = (int)M;
  prm.m_tiles = hidden / kBM;
  prm.n_tiles = (int)(HD / kBN);
  prm.a_mn = 1;
  prm.b_mn = 1;
  prm.ldc = HD;
  prm.M_rows = hidden;
  prm.c32 = dw_o;
  return launch_proj(ta, tb, prm, prof::K_O_PROJ_DWO, stream);
}

uly_status o_proj_launch(int32_t B, int32_t n, int32_t P, int32_t hidden, int32_t H, const void *o,
                         const void *w, void *y, cudaStream_t stream) {
  CUtensorMap ta, tb;
  if (!make_tmap_heads_bf16(&ta, o, kHD, n, P * B * (H / P), kBM) ||
      !make_tmap_rows_bf16(&tb, w, (long long)H * kHD, hidden, kBK, kBN))
    return ULY_ERR_CUDA;
  ProjParams prm = {};
  prm.mode = MODE_OPROJ;
  prm.K = H * kHD;
  prm.tiles_per_b = (n + kBM - 1) / kBM;
  prm.m_tiles = B * prm.tiles_per_b;
  prm.n_tiles = hidden / kBN;
  prm.B = B; prm.n = n; prm.s = n / P; prm.P = P;
  prm.H = H; prm.hl = H / P;
  prm.hidden = hidden;
  prm.y = static_cast<__nv_bfloat16 *>(y);
  prm.err = error_word();
  prm.wait_limit = wait_limit_cycles();
  return launch_proj(ta, tb, prm, prof::K_O_PROJ, stream);
}

}  // namespace uly
