// Local attention forward of every logical rank on the 5th-generation tensor
// cores (Ulysses step 4: "Paralelismul de Secvență Ulysses", section
// "Mecanismul de funcționare Ulysses"; each rank runs ordinary attention on
// its heads over all n positions).  bf16 inputs, fp32 accumulation, head_dim
// 128, causal / doc-causal / no mask, GQA.
//
// One CTA = two 128-row query tiles at the same positions m0..m0+127 of two
// query heads of one GQA group, so both tiles read the same K/V tiles and see
// the same mask: K/V are loaded once for 256 query rows.  When a group has an
// odd number of query heads (MHA: one) the CTA takes one query head: the
// second tile's MMAs and softmax warpgroup are skipped.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: Q tiles once, then K_j, V_j into a 5-slot ring
//   warp 1      TMEM allocator and MMA issuer (one thread):
//                 S_t = Q_t K_j^T          (M=128 N=128 K=128, SS, into TMEM)
//                 O_t += P_t V_j           (M=128 N=128 K=128, P from TMEM, V from smem)
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: one thread
//               per query row reads its S row from TMEM, keeps the running
//               max / sum, writes P (bf16 pairs) back into the TMEM columns of
//               S it has already read, rescales O in TMEM when the max moved by more
//               than 2^8, and finally normalises O and writes O and LSE.
// TMEM: S_0 [0,128) S_1 [128,256) O_0 [256,384) O_1 [384,512) columns; P_t
// occupies columns [0,64) of S_t.  P never touches shared memory, so the
// P V product reads only V from shared memory.
//
// Ordering: s_full[t] is committed after S_j(t), which is issued after
// O_t += P_{j-1} V_{j-1}; a commit tracks every earlier MMA of the thread, so
// when softmax sees S_j it also knows the previous PV finished (O may be
// rescaled).  p_full[t] hands P_j to the MMA warp in two halves (keys
// [0,64) and [64,128)), so the first half of P_j V_j runs while the softmax
// warps compute the second.  S_{j+1}(t) overwrites the
// columns that O_t += P_j V_j reads; both are MMAs of this one issuing thread
// and the tensor core executes them in issue order.
// Every wait is bounded (ULY_ERR_TIMEOUT), no wait can spin forever.
#include "prof.cuh"
#include "sm100.cuh"

namespace uly {

using namespace sm100;

namespace {

constexpr int kBM = 128, kBN = 128, kHD = 128;
constexpr int kThreads = 384;
constexpr int kSlots = 5;
constexpr uint32_t kTileBytes = 128 * 128 * 2;       // one 128 x 128 bf16 tile
constexpr uint32_t kOffQ = 0;                        // 2 tiles
constexpr uint32_t kOffKV = 2 * kTileBytes;          // kSlots tiles
constexpr uint32_t kOffBar = kOffKV + kSlots * kTileBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // barriers + alignment slack
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;            // log2 units
constexpr int kRegsLaunch = 168, kRegsCtl = 88, kRegsSoftmax = 208;
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax == kThreads * kRegsLaunch,
              "register split must use exactly the launch pool");

constexpr uint32_t kIdescS = sm100::idesc_bf16_f32(128, 128, false, false);   // Q K^T
constexpr uint32_t kIdescPV = sm100::idesc_bf16_f32(128, 128, false, true);   // P V (V MN-major)

struct FwdParams {
  __nv_bfloat16 *o;
  float *lse;
  HeadGeom g;
  MaskInfo mk;
  float scale_log2;  // softmax scale * log2(e)
  int *err;          // device error word
  long long wait_limit;  // cycles a pipeline wait may last (wait_limit_cycles())
  int kv_major;          // block order: one KV head at a time (attn_kv_head_major)
};

template <int NTILE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const FwdParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  // barrier indices
  // B_PF + 2t + h: the P of tile t for keys [64h, 64h + 64) is in TMEM
  enum { B_Q = 0, B_KVF = 1, B_KVE = 1 + kSlots, B_SF = 1 + 2 * kSlots, B_PF = B_SF + 2,
         B_OF = B_PF + 4, B_DRAIN = B_OF + 2, B_N = B_DRAIN + 1 };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffBar + 8 * B_N);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffBar + 8 * B_N + 4);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const HeadGeom &g = prm.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int ntile = NTILE;                   // query tiles (heads) per CTA: 2, or 1 for an odd group
  // Blocks start in the order of their linear index (x fastest).  With
  // kv_major that order walks the CTAs of one KV head at a time (its gpp CTAs
  // per query tile, heaviest query tiles first), so the CTAs in flight stream
  // the K/V of one or two KV heads, which stay in L2; without, it takes the
  // heaviest query tiles of every head first.
  int rb, pp, mt;
  if (prm.kv_major) {
    const int gpp = g.group / ntile;             // CTAs per KV head and query tile
    const int nq = gridDim.y;
    const int lin = blockIdx.y * gridDim.x + blockIdx.x;
    const int unit = lin / (gpp * nq), rem = lin - unit * (gpp * nq);   // unit = (r*B + b) * gl + KV head
    mt = nq - 1 - rem / gpp;
    rb = unit / g.gl;
    pp = (unit - rb * g.gl) * gpp + rem % gpp;   // head pair (or head) within the rank
  } else {
    const int per = g.hl / ntile;
    rb = blockIdx.x / per;                       // blockIdx.x = (r*B + b) * per + pp
    pp = blockIdx.x - rb * per;
    mt = gridDim.y - 1 - blockIdx.y;
  }
  const int qhead0 = rb * g.hl + ntile * pp;     // tiles: qhead0 (, qhead0 + 1)
  const int kvhead = rb * g.gl + (ntile * pp) / g.group;
  const int m0 = mt * kBM;

  // KV tiles this query tile touches, and which of them need element masks.
  int lo_first, hi_first, lo_last, hi_last;
  prm.mk.row_range(m0, lo_first, hi_first);
  prm.mk.row_range(min(m0 + kBM - 1, g.n - 1), lo_last, hi_last);
  const int jt0 = lo_first / kBN;
  const int NT = (hi_last >= lo_first) ? hi_last / kBN - jt0 + 1 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_N; ++i) {
      uint32_t cnt = 1;
      if (i >= B_PF && i < B_PF + 4) cnt = 128;
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Registers: the producer / MMA warpgroup (warps 0-3) keeps 88 per thread,
  // each softmax warpgroup gets 208 so a thread can hold a whole 128-column
  // row of S.  128*88 + 256*208 = 384*168, the block's pool at launch.
  if (warp < 4) {
  setmaxnreg_dec<kRegsCtl>();
  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0 && NT > 0) {
      mbar_arrive_expect_tx(bar(B_Q), ntile * kTileBytes);
      for (int t = 0; t < ntile; ++t)
        for (int c = 0; c < 2; ++c)
          tma_load_3d(sb + kOffQ + t * kTileBytes + c * 16384, &tmQ, bar(B_Q), c * 64, m0, qhead0 + t);
      int issued = 0;
      for (int idx = 0; idx < 2 * NT; ++idx) {
        const int slot = idx % kSlots, use = idx / kSlots;
        if (use > 0 && !mbar_wait(bar(B_KVE + slot), (use - 1) & 1, abort_flag, prm.err, prm.wait_limit)) break;
        mbar_arrive_expect_tx(bar(B_KVF + slot), kTileBytes);
        const CUtensorMap *map = (idx & 1) ? &tmV : &tmK;
        const int row0 = (jt0 + idx / 2) * kBN;
        for (int c = 0; c < 2; ++c)
          tma_load_3d(sb + kOffKV + slot * kTileBytes + c * 16384, map, bar(B_KVF + slot), c * 64, row0, kvhead);
        issued = idx + 1;
      }
      // Every copy issued lands before the CTA can exit, also when a consumer
      // gave up waiting for it (older ring entries were consumed, so landed,
      // before their slot was refilled); on the normal path these return at once.
      mbar_wait(bar(B_Q), 0, nullptr, prm.err);
      for (int idx = (issued > kSlots ? issued - kSlots : 0); idx < issued; ++idx)
        mbar_wait(bar(B_KVF + idx % kSlots), (idx / kSlots) & 1, nullptr, prm.err);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0 && NT > 0) {
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag, prm.err, prm.wait_limit);
      tc_fence_after();
      // descriptors of the fixed operands; per-k-step offsets are constants
      uint64_t dq0 = sdesc_sw128(sb + kOffQ, 16, 1024);
      uint64_t dq1 = sdesc_sw128(sb + kOffQ + kTileBytes, 16, 1024);
      // O_t += P_t V over the keys [64h, 64h + 64) (dv: V tile, MN-major)
      auto issue_pv = [&](int t, uint64_t dv, bool first, int h) {
#pragma unroll
        for (int k4 = 0; k4 < kBN / 32; ++k4) {
          const int kk = 4 * h + k4;
          mma_bf16_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, sdesc_add(dv, kk * 2048), kIdescPV,
                      (!first || kk > 0) ? 1u : 0u);
        }
      };
      auto issue_s = [&](int t, uint64_t dk) {
        const uint64_t dq = t ? dq1 : dq0;
#pragma unroll
        for (int kk = 0; kk < kHD / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + t * 128, sdesc_add(dq, koff), sdesc_add(dk, koff), kIdescS, kk > 0 ? 1u : 0u);
        }
      };
      // K/V slots and their phases roll forward (K of tile it at ring index
      // 2 it, V at 2 it + 1); descriptors are computed before the waits so
      // that nothing but MMAs follows a completed wait.
      int slotK = 0, slotV = kSlots - 1;
      uint32_t parK = 0, parV = 1;
      for (int it = 0; ok && it < NT; ++it) {
        // opaque to the compiler, so the per-step descriptors are formed next
        // to their MMAs instead of being hoisted out of the loop
        asm volatile("" : "+l"(dq0), "+l"(dq1));
        const uint64_t dk = sdesc_sw128(sb + kOffKV + slotK * kTileBytes, 16, 1024);
        const uint64_t dv = sdesc_sw128(sb + kOffKV + slotV * kTileBytes, 16384, 1024);   // V: MN-major
        ok = (it > 0) ? mbar_wait2(bar(B_KVF + slotK), parK, bar(B_KVF + slotV), parV, abort_flag, prm.err, prm.wait_limit)
                      : mbar_wait(bar(B_KVF + slotK), parK, abort_flag, prm.err, prm.wait_limit);
        if (!ok) break;
        tc_fence_after();
        for (int t = 0; t < ntile && ok; ++t) {
          if (it > 0) {
            // the first half of P V starts while the softmax still computes the second
            for (int h = 0; h < 2 && ok; ++h) {
              ok = mbar_wait(bar(B_PF + 2 * t + h), (it - 1) & 1, abort_flag, prm.err, prm.wait_limit);
              if (!ok) break;
              tc_fence_after();
              issue_pv(t, dv, it == 1, h);
            }
            if (!ok) break;
          }
          issue_s(t, dk);
          tc_commit(bar(B_SF + t));
        }
        if (!ok) break;
        tc_commit(bar(B_KVE + slotK));
        if (it > 0) tc_commit(bar(B_KVE + slotV));
        slotK += 2;
        if (slotK >= kSlots) { slotK -= kSlots; parK ^= 1u; }
        slotV += 2;
        if (slotV >= kSlots) { slotV -= kSlots; parV ^= 1u; }
      }
      if (ok) {
        // the last tile's V (ring index 2 NT - 1: where slotV has rolled to)
        const uint64_t dv = sdesc_sw128(sb + kOffKV + slotV * kTileBytes, 16384, 1024);
        ok = mbar_wait(bar(B_KVF + slotV), parV, abort_flag, prm.err, prm.wait_limit);
        tc_fence_after();
        for (int t = 0; t < ntile && ok; ++t) {
          for (int h = 0; h < 2 && ok; ++h) {
            ok = mbar_wait(bar(B_PF + 2 * t + h), (NT - 1) & 1, abort_flag, prm.err, prm.wait_limit);
            if (!ok) break;
            tc_fence_after();
            issue_pv(t, dv, NT == 1, h);
          }
          if (!ok) break;
          tc_commit(bar(B_OF + t));
        }
        if (ok) tc_commit(bar(B_KVE + slotV));
      }
      // drain: every MMA issued has completed before TMEM can be released
      tc_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, nullptr, prm.err);
    }
  }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    const int wg = (warp - 4) >> 2;        // query tile 0 or 1
    if (wg < ntile) {
    const int wq = warp & 3;               // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;
    const int i = m0 + row;
    const bool valid = i < g.n;
    int lo_i = 1, hi_i = 0;
    if (valid) prm.mk.row_range(i, lo_i, hi_i);
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + wg * 128;
    const uint32_t tO = tmem + lane_off + 256 + wg * 128;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int it = 0; it < NT; ++it) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SF + wg), it & 1, abort_flag, prm.err, prm.wait_limit));
      if (!ok) break;
      tc_fence_after();
      const int n0 = (jt0 + it) * kBN;
      // the tile needs no element mask when every row of the CTA sees all of it
      const bool full = (n0 >= lo_last) && (n0 + kBN - 1 <= hi_first) && (n0 + kBN <= g.n);
      // One read of the whole 128-column row of S from TMEM.
      uint32_t r[128];
      tmem_ld128(tS, r);
      if (!full) {
#pragma unroll
        for (int x = 0; x < 128; ++x) {
          const int j = n0 + x;
          if (j < lo_i || j > hi_i) r[x] = __float_as_uint(-INFINITY);
        }
      }
      // row maximum of the raw scores (the scale is positive, so the maximum
      // commutes with it); eight independent chains
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = -INFINITY;
#pragma unroll
      for (int x = 0; x < 128; ++x) mx8[x & 7] = fmaxf(mx8[x & 7], __uint_as_float(r[x]));
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * prm.scale_log2;
      const float m_new = fmaxf(m_run, mx);
      const bool had = m_run != -INFINITY;
      const bool rescale = had && (m_new > m_run + kRescaleThreshold);
      if (!had) {
        m_run = m_new;
      } else if (rescale) {
        l_run *= ex2_approx(m_run - m_new);
      }
      if (__any_sync(0xffffffffu, rescale)) {
        const float a = rescale ? ex2_approx(m_run - m_new) : 1.f;
        uint32_t ro[16];
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          tmem_ld16(tO + c * 16, ro);
#pragma unroll
          for (int x = 0; x < 16; ++x) ro[x] = __float_as_uint(__uint_as_float(ro[x]) * a);
          tmem_st16_nowait(tO + c * 16, ro);
          tmem_st_wait();
        }
      }
      if (rescale) m_run = m_new;
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      // P = 2^(s * scale * log2 e - m) as bf16 pairs into TMEM columns [0, 64)
      // of S (already read); eight independent sum chains
      float ls8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) ls8[e] = 0.f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t pk[32];
#pragma unroll
        for (int x = hh * 64; x < hh * 64 + 64; x += 2) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(r[x]), prm.scale_log2, -m_use));
          const float p1 = ex2_approx(fmaf(__uint_as_float(r[x + 1]), prm.scale_log2, -m_use));
          ls8[x & 7] += p0;
          ls8[(x & 7) + 1] += p1;
          pk[(x - hh * 64) >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st32_nowait(tS + hh * 32, pk);
        // hand this half of P to the MMA thread
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(B_PF + 2 * wg + hh));
      }
      l_run += ((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) + ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7]));
    }
    // ---------------------------------------------------------- epilogue
    if (ok && NT > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OF + wg), 0, abort_flag, prm.err, prm.wait_limit));
    tc_fence_after();
    // O goes to the head layout, or straight to the seq layout (the second
    // all-to-all in the epilogue); LSE stays in the head layout
    const long long hrow = (long long)(qhead0 + wg) * g.n + i;
    const long long orow = valid ? g.q_out_row(qhead0 + wg, i) : 0;
    const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
    if (ok && NT > 0) {
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(tO + c * 32, r);
        if (valid) {
          uint4 *dst = reinterpret_cast<uint4 *>(prm.o + orow * kHD + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(r[8 * u + 0]) * inv, __uint_as_float(r[8 * u + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(r[8 * u + 2]) * inv, __uint_as_float(r[8 * u + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(r[8 * u + 4]) * inv, __uint_as_float(r[8 * u + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(r[8 * u + 6]) * inv, __uint_as_float(r[8 * u + 7]) * inv);
            dst[u] = w;
          }
        }
      }
    } else if (valid && NT == 0) {
      uint4 *dst = reinterpret_cast<uint4 *>(prm.o + orow * kHD);
      for (int u = 0; u < kHD / 8; ++u) dst[u] = make_uint4(0, 0, 0, 0);
    }
    if (valid && (ok || NT == 0))
      prm.lse[hrow] = (l_run > 0.f) ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
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

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
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

}  // namespace

// 3-D bf16 map over [heads][n][d] (d = 128) with 64 x 128 x 1 boxes, 128-byte
// swizzle; rows past n read as zero.
bool make_tmap_heads_bf16(CUtensorMap *map, const void *base, int d, int n, int heads, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)n * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                   es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

uly_status attn_bf16_fwd_launch(const uly_attn_desc *d, const HeadGeom &g, const MaskInfo &mk,
                                const void *q, const void *k, const void *v, void *o, float *lse,
                                cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  const int qheads = g.P * g.B * g.hl, kvheads = g.P * g.B * g.gl;
  if (!make_tmap_heads_bf16(&tq, q, kHD, g.n, qheads, 128) ||
      !make_tmap_heads_bf16(&tk, k, kHD, g.n, kvheads, 128) ||
      !make_tmap_heads_bf16(&tv, v, kHD, g.n, kvheads, 128))
    return ULY_ERR_CUDA;
  static std::atomic<uint64_t> optin_devices{0}, optin_devices1{0};
  const int ntile = (g.group & 1) ? 1 : 2;   // two query heads per CTA need an even group
  if (ntile == 2 ? !smem_optin(attn_fwd_sm100_kernel<2>, kSmemBytes, optin_devices)
                 : !smem_optin(attn_fwd_sm100_kernel<1>, kSmemBytes, optin_devices1))
    return ULY_ERR_CUDA;
  FwdParams prm;
  prm.o = static_cast<__nv_bfloat16 *>(o);
  prm.lse = lse;
  prm.g = g;
  prm.mk = mk;
  prm.scale_log2 = g.scale * kLog2e;
  prm.err = error_word();
  prm.wait_limit = wait_limit_cycles();
  dim3 grid(g.P * g.B * (g.hl / ntile), (g.n + kBM - 1) / kBM);
  prm.kv_major = attn_kv_head_major(mk.mask, (long long)grid.y * (g.group / ntile)) ? 1 : 0;
  prof::Scope scope(prof::K_ATTN_FWD_SM100, stream);
  if (ntile == 2)
    attn_fwd_sm100_kernel<2><<<grid, kThreads, kSmemBytes, stream>>>(tq, tk, tv, prm);
  else
    attn_fwd_sm100_kernel<1><<<grid, kThreads, kSmemBytes, stream>>>(tq, tk, tv, prm);
  note_launches(1);
  return last_launch_status();
}

}  // namespace uly
