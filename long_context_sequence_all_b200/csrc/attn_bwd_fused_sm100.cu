// Local attention backward of every logical rank in one pass over the
// (key tile, query tile) pairs: the adjoint of Ulysses step 4
// ("Paralelismul de Secvență Ulysses", section "Mecanismul de funcționare
// Ulysses"; the gradients of sum(O * dO) of each rank's ordinary attention):
//
//   P_ij  = exp(scale q_i.k_j - LSE_i),  dP_ij = dO_i.v_j,  D_i = dO_i.O_i
//   dS_ij = P_ij (dP_ij - D_i)
//   dV_j += P_ij dO_i,   dK_j += scale dS_ij q_i,   dQ_i += scale dS_ij k_j
//
// One CTA owns 128 keys of one KV head (dK, dV accumulate in TMEM over every
// 128-row query tile of every query head of the GQA group that sees those
// keys) and forms each tile's S^T and dP^T once.  Each tile's dQ share over
// the CTA's keys, dQ^T = K^T dS^T, is added into an fp32 accumulator in global
// memory ([query heads][n rounded up to 128][128]; zeroed by the statistics
// kernel, scaled and rounded to bf16 by attn_dq_convert_kernel).  The adds of
// the CTAs that share a query tile meet in L2; their order varies from run to
// run, so dQ is not bitwise repeatable (dK and dV are).
//
// Warp roles (512 threads):
//   warp 0       TMA: K, V once; Q tiles (+ LSE log2 e and D of their rows)
//                in two stages, dO tiles in one; the Q and dO tiles two steps
//                ahead prefetched into L2
//   warp 1       TMEM allocation and the MMA-issuing thread:
//                  S^T  = K Q^T           (SS, M=128 keys, N=128 queries)
//                  dP^T = V dO^T          (SS)
//                  dV  += P^T dO          (TS: P^T from TMEM over S^T)
//                  dQ^T = K^T dS^T        (SS, M=128 head dims, N=128 queries)
//                  dK  += dS^T Q          (SS: dS^T from shared memory)
//   warps 4-11   two compute warpgroups, one key row per thread, each half of
//                the tile's query columns: P^T into TMEM (bf16 pairs over the
//                S^T columns already read), dS^T (bf16) into one of two
//                shared-memory buffers
//   warps 12-15  dQ warpgroup: one head dimension per thread reads the
//                tile's dQ^T row from TMEM and adds it into the accumulator
//                (32 lanes = 32 consecutive floats of one query row per add)
// TMEM: dV [0,128), dK [128,256), S^T / P^T [256,384), dP^T / dQ^T [384,512).
// Issue order per tile t: dV(t), S^T(t+1), dQ^T(t), dK(t), dP^T(t+1); the
// dQ warpgroup empties the dQ^T columns while dK(t) runs, before dP^T(t+1)
// reuses them.  S^T(t+1) overwrites the P^T that dV(t) reads, which relies on
// tcgen05.mma executing in issue order.  Every wait is bounded
// (ULY_ERR_TIMEOUT).
#include "prof.cuh"
#include "sm100.cuh"

namespace uly {

using namespace sm100;

bool make_tmap_heads_bf16(CUtensorMap *map, const void *base, int d, int n, int heads, int box_rows);

namespace {

constexpr int kHD = 128;
constexpr int kThreads = 512;
constexpr float kLog2e = 1.4426950408889634f;

constexpr int kBN = 128;   // keys per CTA
constexpr int kBQ = 128;   // query rows per tile
// Q tiles have two stages: a Q tile is read by S^T (early) and dK (late), so
// its stage is refilled only after the tile's dK.  The LSE and D of the
// tile's rows arrive with it, so the compute warps read both from shared
// memory behind the one barrier they already wait on.  dO tiles have one
// stage: their last reader is dV, near the start of the tile, so the stage is
// released right after it.  dS^T has two buffers, so that a tile's dS^T can be
// written while the previous tile's dQ^T and dK MMAs still read theirs.
constexpr int kQStages = 2, kOStages = 1, kSStages = 2;
static_assert(kSStages == 2, "the dS^T buffer of tile t is t & 1");
constexpr int kPrefetchAhead = 2;
constexpr uint32_t kTile = 128 * 128 * 2;                // one 128 x 128 bf16 tile
constexpr uint32_t kOffK = 0, kOffV = kTile;
constexpr uint32_t kOffQ = 2 * kTile;                    // Q stage s at kOffQ + s * kTile
constexpr uint32_t kOffO = kOffQ + kQStages * kTile;     // dO stage s
constexpr uint32_t kOffS = kOffO + kOStages * kTile;     // dS^T buffer b: [key][query], two 64-query halves
constexpr uint32_t kOffLse = kOffS + kSStages * kTile;   // per Q stage: 128 LSE log2(e)
constexpr uint32_t kOffD = kOffLse + kQStages * kBQ * 4; // per Q stage: 128 D
constexpr uint32_t kEnd = kOffD + kQStages * kBQ * 4;
constexpr uint32_t kBarBytes = 192;
constexpr uint32_t kSmemBytes = 232448;                  // all an SM offers one CTA
// The tiles need a 1024-byte-aligned base.  The barriers go in front of it
// when the alignment gap can hold them, else after the statistics.
constexpr uint32_t kMaxGap = kSmemBytes - kEnd;
static_assert(kEnd + kBarBytes <= kSmemBytes && kMaxGap >= kBarBytes, "fused backward shared memory layout");
constexpr uint32_t kTdV = 0, kTdK = 128, kTS = 256, kTX = 384;

// Register split: control warpgroup, two compute warpgroups, dQ warpgroup.
constexpr int kRegsLaunch = 128;
constexpr int kRegsCtl = 80, kRegsCompute = 144, kRegsDq = 144;
static_assert(128 * (kRegsCtl + 2 * kRegsCompute + kRegsDq) == kThreads * kRegsLaunch,
              "register split must use exactly the launch pool");
static_assert(kRegsCtl < kRegsLaunch && kRegsCompute > kRegsLaunch, "the control warpgroup gives, the compute ones take");

constexpr uint32_t kIdescKK = idesc_bf16_f32(128, 128, false, false);   // A, B K-major
constexpr uint32_t kIdescKM = idesc_bf16_f32(128, 128, false, true);    // B MN-major
constexpr uint32_t kIdescMM = idesc_bf16_f32(128, 128, true, true);     // A, B MN-major

// Fire-and-forget fp32 add into global memory (performed in L2).
__device__ __forceinline__ void red_add_f32(float *p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

struct FusedParams {
  const float *lse2;    // [qheads][n_pad]: LSE log2(e), 0 past n
  const float *Dv;      // [qheads][n_pad]: D, 0 past n
  float *dq_acc;        // [qheads][n_pad][128] fp32, zero on entry
  __nv_bfloat16 *dv;    // [kvheads][n][128]
  __nv_bfloat16 *dk;
  HeadGeom g;
  MaskInfo mk;
  float scale_log2;
  int n_pad;
  int *err;
  long long wait_limit;  // cycles a pipeline wait may last (wait_limit_cycles())
  int kv_major;          // block order: one KV head at a time (attn_kv_head_major)
};

__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_sm100_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                          const FusedParams prm) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t gap = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if (gap > kMaxGap) {   // uniform over the CTA: nothing has been started
    if (threadIdx.x == 0) raise_error(prm.err, ULY_ERR_UNSUPPORTED);
    return;
  }
  uint8_t *smem = smem_raw + gap;
  const uint32_t sb = smem_u32(smem);
  uint8_t *bar_area = (gap >= kBarBytes) ? smem_raw : smem + kEnd;
  uint64_t *bars = reinterpret_cast<uint64_t *>(bar_area);
  enum { B_KV = 0, B_QF = 1, B_QE = B_QF + kQStages, B_OF = B_QE + kQStages, B_OE = B_OF + kOStages,
         B_SF = B_OE + kOStages, B_PS, B_DPF, B_DS, B_DSE, B_DQF = B_DSE + kSStages, B_DQE, B_DONE, B_DRAIN, B_N };
  static_assert(8 * B_N + 8 <= kBarBytes, "barrier area");
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_area + 8 * B_N);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bar_area + 8 * B_N + 4);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const HeadGeom &g = prm.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Blocks start in the order of their linear index (x fastest).  With
  // kv_major that order walks the key tiles of one KV head at a time
  // (earliest, so heaviest under a causal mask, first), so the CTAs in flight
  // read the Q/dO rows and add into the dQ rows of one GQA group's heads,
  // which stay in L2; without, it takes the earliest key tiles of every KV
  // head first.
  int kvh, kt;
  if (prm.kv_major) {
    const int nk = gridDim.y;
    const int lin = blockIdx.y * gridDim.x + blockIdx.x;
    kvh = lin / nk;
    kt = lin - kvh * nk;
  } else {
    kvh = blockIdx.x;
    kt = blockIdx.y;
  }
  const int rb = kvh / g.gl, gg = kvh - rb * g.gl;   // kvh = (r*B + b)*gl + gg
  const int qh_base = rb * g.hl + gg * g.group;  // first query head of the group
  const int n0 = kt * kBN;

  // query rows that see any of the keys [n0, n0+127]
  int lo_a, hi_a, lo_b, hi_b;
  prm.mk.col_range(n0, lo_a, hi_a);
  prm.mk.col_range(min(n0 + kBN - 1, g.n - 1), lo_b, hi_b);
  const int qt0 = lo_a / kBQ;
  const int nqt = (hi_b >= lo_a) ? hi_b / kBQ - qt0 + 1 : 0;
  const int T = nqt * g.group;                   // tiles: head-major

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_N; ++i)
      mbar_init(bar(i), (i == B_PS || i == B_DS) ? 256 : (i == B_DQE ? 128 : 1));
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    setmaxnreg_dec<kRegsCtl>();
    if (warp == 0) {
      // ------------------------------------------------------------ TMA
      if (lane == 0 && T > 0) {
        mbar_arrive_expect_tx(bar(B_KV), 2 * kTile);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(sb + kOffK + c * 16384, &tmK, bar(B_KV), c * 64, n0, kvh);
          tma_load_3d(sb + kOffV + c * 16384, &tmV, bar(B_KV), c * 64, n0, kvh);
        }
        int issued_q = 0, issued_o = 0;
        for (int t = 0; t < T; ++t) {
          const int e = t / nqt, i0 = (qt0 + t - e * nqt) * kBQ;
          const long long srow = (long long)(qh_base + e) * prm.n_pad + i0;
          const int sq = t % kQStages, uq = t / kQStages;
          if (uq > 0 && !mbar_wait(bar(B_QE + sq), (uq - 1) & 1, abort_flag, prm.err, prm.wait_limit)) break;
          mbar_arrive_expect_tx(bar(B_QF + sq), kTile + 2 * kBQ * 4);
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sb + kOffQ + sq * kTile + c * 16384, &tmQ, bar(B_QF + sq), c * 64, i0, qh_base + e);
          bulk_load(sb + kOffLse + sq * kBQ * 4, prm.lse2 + srow, kBQ * 4, bar(B_QF + sq));
          bulk_load(sb + kOffD + sq * kBQ * 4, prm.Dv + srow, kBQ * 4, bar(B_QF + sq));
          issued_q = t + 1;
          // the Q and dO tiles kPrefetchAhead tiles on, into L2 (their loads
          // otherwise wait on L2 misses behind the dQ reduce-adds)
          if (kPrefetchAhead > 0 && t + kPrefetchAhead < T) {
            const int tp = t + kPrefetchAhead, ep = tp / nqt, ip = (qt0 + tp - ep * nqt) * kBQ;
            for (int c = 0; c < 2; ++c) {
              tma_prefetch_l2_3d(&tmQ, c * 64, ip, qh_base + ep);
              tma_prefetch_l2_3d(&tmO, c * 64, ip, qh_base + ep);
            }
          }
          const int so = t % kOStages, uo = t / kOStages;
          if (uo > 0 && !mbar_wait(bar(B_OE + so), (uo - 1) & 1, abort_flag, prm.err, prm.wait_limit)) break;
          mbar_arrive_expect_tx(bar(B_OF + so), kTile);
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sb + kOffO + so * kTile + c * 16384, &tmO, bar(B_OF + so), c * 64, i0, qh_base + e);
          issued_o = t + 1;
        }
        // Every copy issued lands before the CTA can exit, also when a consumer
        // gave up waiting for it (older stages were consumed, so landed,
        // before they were refilled); on the normal path these return at once.
        mbar_wait(bar(B_KV), 0, nullptr, prm.err);
        for (int t = (issued_q > kQStages ? issued_q - kQStages : 0); t < issued_q; ++t)
          mbar_wait(bar(B_QF + t % kQStages), (t / kQStages) & 1, nullptr, prm.err);
        for (int t = (issued_o > kOStages ? issued_o - kOStages : 0); t < issued_o; ++t)
          mbar_wait(bar(B_OF + t % kOStages), (t / kOStages) & 1, nullptr, prm.err);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA
      if (lane == 0 && T > 0) {
        bool ok = mbar_wait(bar(B_KV), 0, abort_flag, prm.err, prm.wait_limit);
        uint64_t dK = sdesc_sw128(sb + kOffK, 16, 1024), dV = sdesc_sw128(sb + kOffV, 16, 1024);
        uint64_t dKt = sdesc_sw128(sb + kOffK, 16384, 1024);   // K^T (A of dQ^T): MN-major
        uint64_t dSb = sdesc_sw128(sb + kOffS, 16384, 1024);   // dS^T (B of dQ^T): MN-major
        uint64_t dSa = sdesc_sw128(sb + kOffS, 16, 1024);      // dS^T (A of dK): K-major
        auto issue_s = [&](uint64_t dQ) {
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16_ss(tmem + kTS, sdesc_add(dK, ko), sdesc_add(dQ, ko), kIdescKK, kk > 0);
          }
          tc_commit(bar(B_SF));
        };
        auto issue_dp = [&](uint64_t dO) {
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16_ss(tmem + kTX, sdesc_add(dV, ko), sdesc_add(dO, ko), kIdescKK, kk > 0);
          }
          tc_commit(bar(B_DPF));
        };
        if (ok) ok = mbar_wait2(bar(B_QF), 0, bar(B_OF), 0, abort_flag, prm.err, prm.wait_limit);
        if (ok) {
          tc_fence_after();
          issue_s(sdesc_sw128(sb + kOffQ, 16, 1024));
          issue_dp(sdesc_sw128(sb + kOffO, 16, 1024));
        }
        // Stages and parities roll forward; every descriptor of an iteration
        // is computed before its waits, so only MMAs follow a completed wait.
        int sq = 0, so = 0;
        uint32_t pq = 0, po = 0;
        for (int t = 0; ok && t < T; ++t) {
          // Opaque to the compiler: the per-step descriptors (base + a constant)
          // are then formed next to their MMA instead of being hoisted out of
          // the loop into ~80 live registers.
          asm volatile("" : "+l"(dK), "+l"(dV), "+l"(dKt), "+l"(dSb), "+l"(dSa));
          const bool more = t + 1 < T;
          const int sq1 = (sq + 1 == kQStages) ? 0 : sq + 1, so1 = (so + 1 == kOStages) ? 0 : so + 1;
          const uint32_t pq1 = (sq1 == 0) ? (pq ^ 1u) : pq, po1 = (so1 == 0) ? (po ^ 1u) : po;
          const uint64_t dOm = sdesc_sw128(sb + kOffO + so * kTile, 16384, 1024);   // dV: B = dO, MN-major
          const uint64_t dQm = sdesc_sw128(sb + kOffQ + sq * kTile, 16384, 1024);   // dK: B = Q, MN-major
          const uint64_t dQn = sdesc_sw128(sb + kOffQ + sq1 * kTile, 16, 1024);     // next S^T: B = next Q
          const uint64_t dOn = sdesc_sw128(sb + kOffO + so1 * kTile, 16, 1024);     // next dP^T: B = next dO
          // dV += P^T dO_t: A from TMEM (query columns [0,64) in the S^T
          // columns [0,32), [64,128) in [64,96))
          ok = mbar_wait(bar(B_PS), t & 1, abort_flag, prm.err, prm.wait_limit);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBQ / 16; ++kk) {
            const uint32_t acol = (kk >> 2) * 64 + (kk & 3) * 8;
            mma_bf16_ts(tmem + kTdV, tmem + kTS + acol, sdesc_add(dOm, kk * 2048), kIdescKM,
                        (t > 0 || kk > 0) ? 1u : 0u);
          }
          // dO_t has been read by its two MMAs (dP^T earlier, dV now)
          tc_commit(bar(B_OE + so));
          // the next tile's S^T over this tile's P^T (after the dV MMA in issue order)
          if (more) {
            ok = mbar_wait(bar(B_QF + sq1), pq1, abort_flag, prm.err, prm.wait_limit);
            if (!ok) break;
            tc_fence_after();
            issue_s(dQn);
          }
          // dS^T of the tile is in shared memory and the dP^T columns are read
          ok = mbar_wait(bar(B_DS), t & 1, abort_flag, prm.err, prm.wait_limit);
          if (!ok) break;
          tc_fence_after();
          // dQ^T = K^T dS^T into the dP^T columns: M = head dims, N = queries,
          // K = the CTA's keys (16 rows of both tiles per step)
          const uint32_t sbo = (uint32_t)(t & 1) * kTile;   // this tile's dS^T buffer
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            mma_bf16_ss(tmem + kTX, sdesc_add(dKt, kk * 2048), sdesc_add(dSb, sbo + kk * 2048), kIdescMM, kk > 0);
          tc_commit(bar(B_DQF));
          // dK += dS^T Q_t: A = dS^T (K-major: the queries of a key row)
#pragma unroll
          for (int kk = 0; kk < kBQ / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16_ss(tmem + kTdK, sdesc_add(dSa, sbo + ko), sdesc_add(dQm, kk * 2048), kIdescKM,
                        (t > 0 || kk > 0) ? 1u : 0u);
          }
          // tile t's Q stage and dS^T buffer are free once dK is done
          tc_commit(bar(B_QE + sq));
          tc_commit(bar(B_DSE + (t & 1)));
          if (more) {
            // the next dP^T reuses the dQ^T columns once the dQ warpgroup has read them
            ok = mbar_wait2(bar(B_DQE), t & 1, bar(B_OF + so1), po1, abort_flag, prm.err, prm.wait_limit);
            if (!ok) break;
            tc_fence_after();
            issue_dp(dOn);
          }
          sq = sq1; so = so1; pq = pq1; po = po1;
        }
        if (ok) tc_commit(bar(B_DONE));
        // every MMA issued has completed before TMEM can be released
        tc_commit(bar(B_DRAIN));
        mbar_wait(bar(B_DRAIN), 0, nullptr, prm.err);
      }
    }
  } else if (warp < 12) {
    // ---------------------------------------------------------- compute
    setmaxnreg_inc<kRegsCompute>();
    const int w = (warp - 4) >> 2, wq = warp & 3;  // w: query columns [64w, 64w + 64)
    const int row = wq * 32 + lane;                // key row within the tile
    const int j = n0 + row;
    int lo_j = 1, hi_j = 0;
    if (j < g.n) prm.mk.col_range(j, lo_j, hi_j);
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + kTS + 64 * w, tP = tmem + lane_off + kTX + 64 * w;
    // this thread's row of dS^T: 128 bytes in the warpgroup's 64-query half
    const uint32_t ds_row0 = sb + kOffS + w * 16384 + row * 128;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int e = t / nqt, i0 = (qt0 + t - e * nqt) * kBQ + 64 * w;  // this warpgroup's first query row
      const int sq = t % kQStages;
      const float *lsm = reinterpret_cast<const float *>(smem + kOffLse + sq * kBQ * 4) + 64 * w;
      // D of this warpgroup's 64 query rows, staged with the Q tile
      const float4 *d4 = reinterpret_cast<const float4 *>(smem + kOffD + sq * kBQ * 4) + 16 * w;
      // P^T over this warpgroup's first 32 columns of S^T
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_QF + sq), (t / kQStages) & 1, abort_flag, prm.err, prm.wait_limit) &&
                                       mbar_wait(bar(B_SF), t & 1, abort_flag, prm.err, prm.wait_limit));
      if (!ok) break;
      tc_fence_after();
      const bool full = (i0 >= n0 + kBN - 1) && (i0 + 63 <= hi_a) && (i0 + 64 <= g.n) && (n0 + kBN <= g.n);
      uint32_t r[64];
      tmem_ld64(tS, r);
      // masked scores become -inf (exponential 0) before the exponentials, so
      // that their loop has no branch and its MUFU latencies overlap freely
      if (!full) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (i0 + c < lo_j || i0 + c > hi_j) r[c] = __float_as_uint(-INFINITY);
      }
      uint32_t pp[32];
      // LSE log2(e) of the 64 query rows: one broadcast 16-byte shared-memory
      // load per 4 columns
      const float4 *l4 = reinterpret_cast<const float4 *>(lsm);
#pragma unroll
      for (int c = 0; c < 64; c += 4) {
        const float4 L = l4[c >> 2];
        const float p0 = ex2_approx(fmaf(__uint_as_float(r[c]), prm.scale_log2, -L.x));
        const float p1 = ex2_approx(fmaf(__uint_as_float(r[c + 1]), prm.scale_log2, -L.y));
        const float p2 = ex2_approx(fmaf(__uint_as_float(r[c + 2]), prm.scale_log2, -L.z));
        const float p3 = ex2_approx(fmaf(__uint_as_float(r[c + 3]), prm.scale_log2, -L.w));
        r[c] = __float_as_uint(p0);
        r[c + 1] = __float_as_uint(p1);
        r[c + 2] = __float_as_uint(p2);
        r[c + 3] = __float_as_uint(p3);
        pp[c >> 1] = pack_bf16x2(p0, p1);
        pp[(c >> 1) + 1] = pack_bf16x2(p2, p3);
      }
      tmem_st32_nowait(tS, pp);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_PS));
      // dS^T = P^T (dP^T - D) into shared memory
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DPF), t & 1, abort_flag, prm.err, prm.wait_limit));
      if (!ok) break;
      tc_fence_after();
      uint32_t dp[64];
      tmem_ld64(tP, dp);
      uint32_t dd[32];
#pragma unroll
      for (int c = 0; c < 64; c += 4) {
        const float4 dq4 = d4[c >> 2];
        dd[c >> 1] = pack_bf16x2(__uint_as_float(r[c]) * (__uint_as_float(dp[c]) - dq4.x),
                                 __uint_as_float(r[c + 1]) * (__uint_as_float(dp[c + 1]) - dq4.y));
        dd[(c >> 1) + 1] = pack_bf16x2(__uint_as_float(r[c + 2]) * (__uint_as_float(dp[c + 2]) - dq4.z),
                                       __uint_as_float(r[c + 3]) * (__uint_as_float(dp[c + 3]) - dq4.w));
      }
      // the dQ^T and dK MMAs of the tile two back have read this buffer
      if (t >= kSStages) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DSE + (t & 1)), ((t >> 1) - 1) & 1, abort_flag, prm.err,
                                               prm.wait_limit));
        if (!ok) break;
      }
      const uint32_t ds_row = ds_row0 + (uint32_t)(t & 1) * kTile;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(ds_row + ((uint32_t)(c ^ (row & 7)) << 4), dd[4 * c], dd[4 * c + 1], dd[4 * c + 2],
                     dd[4 * c + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(B_DS));
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK (scaled)
    if (ok && T > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DONE), 0, abort_flag, prm.err, prm.wait_limit));
    tc_fence_after();
    __nv_bfloat16 *outp = (w == 0) ? prm.dv : prm.dk;
    const float mul = (w == 0) ? 1.f : g.scale;
    const long long orow = (j < g.n) ? g.kv_out_row(kvh, j) : 0;
    if (ok && T > 0) {
      uint32_t rr[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(tmem + lane_off + (w == 0 ? kTdV : kTdK) + c * 32, rr);
        if (j < g.n) {
          uint4 *dptr = reinterpret_cast<uint4 *>(outp + orow * kHD + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(rr[8 * u + 0]) * mul, __uint_as_float(rr[8 * u + 1]) * mul);
            v.y = pack_bf16x2(__uint_as_float(rr[8 * u + 2]) * mul, __uint_as_float(rr[8 * u + 3]) * mul);
            v.z = pack_bf16x2(__uint_as_float(rr[8 * u + 4]) * mul, __uint_as_float(rr[8 * u + 5]) * mul);
            v.w = pack_bf16x2(__uint_as_float(rr[8 * u + 6]) * mul, __uint_as_float(rr[8 * u + 7]) * mul);
            dptr[u] = v;
          }
        }
      }
    } else if (T == 0 && j < g.n) {
      uint4 *dptr = reinterpret_cast<uint4 *>(outp + orow * kHD);
      for (int u = 0; u < kHD / 8; ++u) dptr[u] = make_uint4(0, 0, 0, 0);
    }
  } else {
    // -------------------------------------------------------------- dQ
    if constexpr (kRegsDq > kRegsLaunch) setmaxnreg_inc<kRegsDq>();
    else if constexpr (kRegsDq < kRegsLaunch) setmaxnreg_dec<kRegsDq>();
    const int wq = warp & 3;
    const int dcol = wq * 32 + lane;               // head dimension = TMEM lane of dQ^T
    const uint32_t tX = tmem + ((uint32_t)(wq * 32) << 16) + kTX;
    for (int t = 0; t < T; ++t) {
      const int e = t / nqt, i0 = (qt0 + t - e * nqt) * kBQ;
      float *dst = prm.dq_acc + ((long long)(qh_base + e) * prm.n_pad + i0) * kHD + dcol;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_DQF), t & 1, abort_flag, prm.err, prm.wait_limit))) break;
      tc_fence_after();
      // the whole dQ^T row (128 queries) in one read, so that the columns are
      // handed back to the next dP^T before any of the adds is issued
      uint32_t v[128];
      tmem_ld64x2(tX, tX + 64, v);
      tc_fence_before();
      mbar_arrive(bar(B_DQE));
#pragma unroll
      for (int q = 0; q < 128; ++q) red_add_f32(dst + q * kHD, __uint_as_float(v[q]));
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

// dQ = scale * accumulator, rounded to bf16, in the head or the seq layout:
// two rows per warp, 16-byte stores.
__global__ void __launch_bounds__(256) attn_dq_convert_kernel(const float *__restrict__ acc,
                                                              __nv_bfloat16 *__restrict__ dq, HeadGeom g,
                                                              int n_pad, long long rows_pad) {
  const long long r = (long long)blockIdx.x * 16 + (threadIdx.x >> 4);
  const int l = threadIdx.x & 15;
  if (r >= rows_pad) return;
  const long long h = r / n_pad;
  const int i = (int)(r - h * n_pad);
  if (i >= g.n) return;
  const float scale = g.scale;
  const float4 *src = reinterpret_cast<const float4 *>(acc + r * kHD) + 2 * l;
  const float4 a = __ldcs(src), b = __ldcs(src + 1);
  uint4 o;
  o.x = pack_bf16x2(a.x * scale, a.y * scale);
  o.y = pack_bf16x2(a.z * scale, a.w * scale);
  o.z = pack_bf16x2(b.x * scale, b.y * scale);
  o.w = pack_bf16x2(b.z * scale, b.w * scale);
  reinterpret_cast<uint4 *>(dq + g.q_out_row(h, i) * kHD)[l] = o;
}

}  // namespace

// The fused launch: the statistics kernel has written D, LSE log2(e) and
// zeroed dq_acc; this runs the fused kernel and the dQ conversion.
uly_status attn_bf16_bwd_fused_launch(const HeadGeom &g, const MaskInfo &mk, const void *q, const void *k,
                                      const void *v, const void *dout, void *dq, void *dk, void *dv,
                                      const float *Dv, const float *L2, float *dq_acc, int n_pad,
                                      cudaStream_t stream) {
  const int qheads = g.P * g.B * g.hl, kvheads = g.P * g.B * g.gl;
  CUtensorMap mK, mV, mQ, mO;
  if (!make_tmap_heads_bf16(&mK, k, kHD, g.n, kvheads, 128) || !make_tmap_heads_bf16(&mV, v, kHD, g.n, kvheads, 128) ||
      !make_tmap_heads_bf16(&mQ, q, kHD, g.n, qheads, 128) || !make_tmap_heads_bf16(&mO, dout, kHD, g.n, qheads, 128))
    return ULY_ERR_CUDA;
  static std::atomic<uint64_t> optin_devices{0};
  if (!smem_optin(attn_bwd_sm100_kernel, kSmemBytes, optin_devices)) return ULY_ERR_CUDA;
  FusedParams prm;
  prm.lse2 = L2;
  prm.Dv = Dv;
  prm.dq_acc = dq_acc;
  prm.dv = static_cast<__nv_bfloat16 *>(dv);
  prm.dk = static_cast<__nv_bfloat16 *>(dk);
  prm.g = g;
  prm.mk = mk;
  prm.scale_log2 = g.scale * kLog2e;
  prm.n_pad = n_pad;
  prm.err = error_word();
  prm.wait_limit = wait_limit_cycles();
  prm.kv_major = attn_kv_head_major(mk.mask, (g.n + kBN - 1) / kBN) ? 1 : 0;
  {
    prof::Scope scope(prof::K_ATTN_BWD_SM100, stream);
    attn_bwd_sm100_kernel<<<dim3(kvheads, (g.n + kBN - 1) / kBN), kThreads, kSmemBytes, stream>>>(mK, mV, mQ, mO,
                                                                                                 prm);
  }
  const long long rows_pad = (long long)qheads * n_pad;
  {
    prof::Scope scope(prof::K_ATTN_DQ_CONVERT, stream);
    attn_dq_convert_kernel<<<(unsigned)((rows_pad + 15) / 16), 256, 0, stream>>>(
        dq_acc, static_cast<__nv_bfloat16 *>(dq), g, n_pad, rows_pad);
  }
  note_launches(2);
  return last_launch_status();
}

}  // namespace uly
