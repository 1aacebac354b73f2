// Local attention backward of every logical rank on the 5th-generation tensor
// cores (the adjoint of Ulysses step 4; the gradients of sum(O * dO)):
//
//   P_ij  = exp(scale * q_i.k_j - LSE_i)          (recomputed, never stored)
//   dP_ij = dO_i . v_j,   D_i = dO_i . O_i,   dS_ij = P_ij (dP_ij - D_i)
//   dV_j  = sum_i P_ij dO_i          dK_j = scale * sum_i dS_ij q_i
//   dQ_i  = scale * sum_j dS_ij k_j
// with dK, dV summed over the query heads that share a KV head (GQA).
//
// Three launches, all deterministic (no atomics):
//  1. D_i = <dO_i, O_i> and LSE_i log2(e) into arrays whose query rows are
//     padded to a multiple of 128 (zeros past n), so that every 128-row tile
//     of them is one aligned 512-byte block (HBM-bound)
//  2. dK/dV kernel, KV-stationary: a CTA owns 128 keys of one KV head and
//     visits every 128-row query tile (of every query head of the group) that
//     sees them; the two compute warpgroups split each tile's query columns:
//       S^T  = K Q^T,  dP^T = V dO^T          (M=128 keys, N=128 queries, K=128)
//       dV  += P^T dO, dK  += dS^T Q           (M=128 keys, N=128,      K=128)
//     P^T and dS^T stay in TMEM over S^T / dP^T (A of dV and dK), as do dK
//     and dV; Q tiles have three shared-memory stages, dO tiles two.
//  3. dQ kernel, query-stationary: a CTA owns 128 query rows of one head
//     with Q and dO resident in TMEM, and streams K/V tiles of 128 keys:
//       S = Q K^T, dP = dO V^T (M=128, N=128, K=128, A from TMEM)
//       dQ += dS K             (M=128, N=128, K=128, dS from TMEM)
//     The next tile's S is issued as soon as the current S has been read.
//
// TMA loads with 128-byte swizzle feed shared memory; one thread issues all
// MMAs; every wait is bounded (ULY_ERR_TIMEOUT).
#include "prof.cuh"
#include "sm100.cuh"

namespace uly {

using namespace sm100;

bool make_tmap_heads_bf16(CUtensorMap *map, const void *base, int d, int n, int heads, int box_rows);

namespace {

constexpr int kHD = 128;
constexpr int kThreads = 384;
constexpr float kLog2e = 1.4426950408889634f;

constexpr int kRegsLaunch = 168;
constexpr int kRegsCtlKV = 120, kRegsComputeKV = 192;  // dK/dV kernel
constexpr int kRegsCtlQ = 120, kRegsComputeQ = 192;    // dQ kernel
static_assert(128 * kRegsCtlKV + 256 * kRegsComputeKV == kThreads * kRegsLaunch &&
                  128 * kRegsCtlQ + 256 * kRegsComputeQ == kThreads * kRegsLaunch,
              "register split must use exactly the launch pool");

constexpr uint32_t kIdescN128 = idesc_bf16_f32(128, 128, false, false);  // K-major A and B, N = 128
constexpr uint32_t kIdescN128MN = idesc_bf16_f32(128, 128, false, true); // B MN-major, N = 128

struct BwdParams {
  const __nv_bfloat16 *q;     // [qheads][n][d] (dQ kernel: Q rows go into TMEM)
  const __nv_bfloat16 *dout;  // [qheads][n][d]
  const float *lse2;  // [qheads][n_pad]: LSE log2(e), 0 past n
  const float *Dv;    // [qheads][n_pad]: D, 0 past n
  __nv_bfloat16 *out0;  // dkdv: dV, dq: dQ
  __nv_bfloat16 *out1;  // dkdv: dK
  HeadGeom g;
  MaskInfo mk;
  float scale_log2;
  int n_pad;          // n rounded up to a multiple of 128
  int *err;
  long long wait_limit;  // cycles a pipeline wait may last (wait_limit_cycles())
  int kv_major;       // block order: one KV head at a time (attn_kv_head_major)
};

// D_i = <dO_i, O_i> and LSE_i log2(e) of every query row (two rows per warp,
// 16-byte loads), written to the padded per-head arrays; rows n..n_pad-1 get 0,
// rows that see no key an LSE of +inf.
// dq_acc (fused backward only, else null): the row's 128 fp32 dQ accumulators
// are zeroed here, so the fused kernel finds them cleared.
// O is read in the head layout, or in the seq layout when g.out_seq (the
// layout the forward wrote it in); dO and LSE are in the head layout.
__global__ void __launch_bounds__(256) attn_bwd_stats_kernel(const __nv_bfloat16 *__restrict__ o,
                                                             const __nv_bfloat16 *__restrict__ dout,
                                                             const float *__restrict__ lse,
                                                             float *__restrict__ Dpad,
                                                             float *__restrict__ L2pad, float *__restrict__ dq_acc,
                                                             HeadGeom g, int n_pad, long long rows_pad) {
  const int n = g.n;
  const long long r = (long long)blockIdx.x * 16 + (threadIdx.x >> 4);
  const int l = threadIdx.x & 15;
  if (dq_acc && r < rows_pad) {
    float4 *z = reinterpret_cast<float4 *>(dq_acc + r * kHD) + 2 * l;
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const long long h = r / n_pad;
  const int i = (int)(r - h * n_pad);
  const bool valid = r < rows_pad && i < n;
  float acc = 0.f;
  if (valid) {
    const long long src = (h * n + i) * kHD;
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(o + g.q_out_row(h, i) * kHD) + l);
    const uint4 b = __ldg(reinterpret_cast<const uint4 *>(dout + src) + l);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&av[u]));
      const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&bv[u]));
      acc = fmaf(fa.x, fb.x, acc);
      acc = fmaf(fa.y, fb.y, acc);
    }
  }
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (l == 0 && r < rows_pad) {
    Dpad[r] = acc;
    // a row that sees no key (forward LSE -inf) gets +inf: every exponential
    // of the row, masked or not, is then exactly 0
    const float lv = valid ? __ldg(lse + h * n + i) : 0.f;
    L2pad[r] = valid ? (lv == -INFINITY ? INFINITY : lv * kLog2e) : 0.f;
  }
}

// ============================================================== dK / dV
// One CTA = 128 keys of one KV head; it visits every 128-row query tile (of
// every query head of the group) that sees them:
//   S^T  = K Q^T,  dP^T = V dO^T   (M=128 keys, N=128 queries, K=128; A and B from smem)
//   dV  += P^T dO, dK  += dS^T Q    (M=128, N=128, K=128 queries; A from TMEM)
// The two compute warpgroups split the 128 query columns of a tile (64
// each); each writes its half of P^T and dS^T (bf16 pairs) over TMEM columns
// of S^T / dP^T that it has itself already read, so shared memory holds only
// operand tiles: K, V, three Q stages (a Q tile is needed until the tile's dK
// MMA, and the next tiles' Q loads must not sit on the critical path) and two
// dO stages.  Each tile's LSE log2(e) and D travel with its Q and dO tiles.
// TMEM: dV [0,128), dK [128,256), S^T / P^T [256,384), dP^T / dS^T [384,512).
// The next tile's S^T is issued right after this tile's dV MMA and its dP^T
// right after the dK MMA: they overwrite the P^T / dS^T those MMAs read, which
// relies on tcgen05.mma executing in issue order.
namespace kv {
constexpr int kBN = 128;   // keys per CTA
constexpr int kBQ = 128;   // query rows per tile
constexpr int kQStages = 3, kOStages = 2;
constexpr uint32_t kTile = 128 * 128 * 2;          // one 128 x 128 bf16 tile
constexpr uint32_t kOffK = 0, kOffV = kTile;
constexpr uint32_t kOffQ = 2 * kTile;                          // Q stage s at kOffQ + s * kTile
constexpr uint32_t kOffO = kOffQ + kQStages * kTile;           // dO stage s at kOffO + s * kTile
constexpr uint32_t kOffLse = kOffO + kOStages * kTile;         // per Q stage: 128 LSE log2(e)
constexpr uint32_t kOffD = kOffLse + kQStages * kBQ * 4;       // per dO stage: 128 D
constexpr uint32_t kEnd = kOffD + kOStages * kBQ * 4;
constexpr uint32_t kBarBytes = 160;
constexpr uint32_t kSmemBytes = 232448;                        // all an SM offers one CTA
// The tiles need a 1024-byte-aligned base.  The barriers go in front of it
// when the alignment gap can hold them, else after the statistics; a gap
// larger than kMaxGap would not fit and is reported (ULY_ERR_UNSUPPORTED).
constexpr uint32_t kMaxGap = kSmemBytes - kEnd;
static_assert(kEnd + kBarBytes <= kSmemBytes && kMaxGap >= kBarBytes, "dK/dV shared memory layout");
constexpr uint32_t kTdV = 0, kTdK = 128, kTS = 256, kTP = 384;
}  // namespace kv

__global__ void __launch_bounds__(kThreads, 1)
    attn_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                           const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                           const BwdParams prm) {
  using namespace kv;
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
         B_SF = B_OE + kOStages, B_PS, B_DPF, B_DS, B_DONE, B_DRAIN, B_N };
  static_assert(8 * B_N + 8 <= kBarBytes, "barrier area");
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_area + 8 * B_N);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bar_area + 8 * B_N + 4);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const HeadGeom &g = prm.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Blocks start in the order of their linear index (x fastest): with
  // kv_major the key tiles of one KV head at a time, else those of every KV
  // head side by side; earliest keys (heaviest) first either way.
  int kvh, kt;
  if (prm.kv_major) {
    const int lin = blockIdx.y * gridDim.x + blockIdx.x;
    kvh = lin / gridDim.y;
    kt = lin - kvh * gridDim.y;
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
    for (int i = 0; i < B_N; ++i) mbar_init(bar(i), (i == B_PS || i == B_DS) ? 256 : 1);
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
  // Registers: producer / MMA warpgroup 120 per thread, the two compute
  // warpgroups 192 (a thread holds 64 values of P^T and 64 of dP^T).

  if (warp < 4) {
  setmaxnreg_dec<kRegsCtlKV>();
  if (warp == 0) {
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
        // Q tile and its LSE
        const int sq = t % kQStages, uq = t / kQStages;
        if (uq > 0 && !mbar_wait(bar(B_QE + sq), (uq - 1) & 1, abort_flag, prm.err, prm.wait_limit)) break;
        mbar_arrive_expect_tx(bar(B_QF + sq), kTile + kBQ * 4);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(sb + kOffQ + sq * kTile + c * 16384, &tmQ, bar(B_QF + sq), c * 64, i0, qh_base + e);
        bulk_load(sb + kOffLse + sq * kBQ * 4, prm.lse2 + srow, kBQ * 4, bar(B_QF + sq));
        issued_q = t + 1;
        // dO tile and its D
        const int so = t % kOStages, uo = t / kOStages;
        if (uo > 0 && !mbar_wait(bar(B_OE + so), (uo - 1) & 1, abort_flag, prm.err, prm.wait_limit)) break;
        mbar_arrive_expect_tx(bar(B_OF + so), kTile + kBQ * 4);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(sb + kOffO + so * kTile + c * 16384, &tmO, bar(B_OF + so), c * 64, i0, qh_base + e);
        bulk_load(sb + kOffD + so * kBQ * 4, prm.Dv + srow, kBQ * 4, bar(B_OF + so));
        issued_o = t + 1;
      }
      // every copy issued lands before the CTA can exit (see the forward)
      mbar_wait(bar(B_KV), 0, nullptr, prm.err);
      for (int t = (issued_q > kQStages ? issued_q - kQStages : 0); t < issued_q; ++t)
        mbar_wait(bar(B_QF + t % kQStages), (t / kQStages) & 1, nullptr, prm.err);
      for (int t = (issued_o > kOStages ? issued_o - kOStages : 0); t < issued_o; ++t)
        mbar_wait(bar(B_OF + t % kOStages), (t / kOStages) & 1, nullptr, prm.err);
    }
  } else if (warp == 1) {
    if (lane == 0 && T > 0) {
      bool ok = mbar_wait(bar(B_KV), 0, abort_flag, prm.err, prm.wait_limit);
      const uint64_t dK = sdesc_sw128(sb + kOffK, 16, 1024), dV = sdesc_sw128(sb + kOffV, 16, 1024);
      // S^T = K Q^T into the S^T columns; dP^T = V dO^T into the dP^T columns
      auto issue_s = [&](uint64_t dQ) {
#pragma unroll
        for (int kk = 0; kk < kHD / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + kTS, sdesc_add(dK, ko), sdesc_add(dQ, ko), kIdescN128, kk > 0);
        }
        tc_commit(bar(B_SF));
      };
      auto issue_dp = [&](uint64_t dO) {
#pragma unroll
        for (int kk = 0; kk < kHD / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + kTP, sdesc_add(dV, ko), sdesc_add(dO, ko), kIdescN128, kk > 0);
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
      // is computed before its waits, so that nothing but the MMAs follows a
      // completed wait (the issue queue is shallow, so any latency there idles
      // the tensor pipe).  The dV group waits at one point for P^T and the
      // next Q tile.
      int sq = 0, so = 0;
      uint32_t pq = 0, po = 0;
      for (int t = 0; ok && t < T; ++t) {
        const bool more = t + 1 < T;
        const int sq1 = (sq + 1 == kQStages) ? 0 : sq + 1, so1 = (so + 1 == kOStages) ? 0 : so + 1;
        const uint32_t pq1 = (sq1 == 0) ? (pq ^ 1u) : pq, po1 = (so1 == 0) ? (po ^ 1u) : po;
        const uint64_t dOm = sdesc_sw128(sb + kOffO + so * kTile, 16384, 1024);   // dV: B = dO, MN-major
        const uint64_t dQm = sdesc_sw128(sb + kOffQ + sq * kTile, 16384, 1024);   // dK: B = Q, MN-major
        const uint64_t dQn = sdesc_sw128(sb + kOffQ + sq1 * kTile, 16, 1024);     // next S^T: B = next Q
        const uint64_t dOn = sdesc_sw128(sb + kOffO + so1 * kTile, 16, 1024);     // next dP^T: B = next dO
        // dV += P^T dO_t: A from TMEM (query columns [0,64) in the S^T
        // columns [0,32), [64,128) in [64,96))
        ok = more ? mbar_wait2(bar(B_PS), t & 1, bar(B_QF + sq1), pq1, abort_flag, prm.err, prm.wait_limit)
                  : mbar_wait(bar(B_PS), t & 1, abort_flag, prm.err, prm.wait_limit);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBQ / 16; ++kk) {
          const uint32_t acol = (kk >> 2) * 64 + (kk & 3) * 8;
          mma_bf16_ts(tmem + kTdV, tmem + kTS + acol, sdesc_add(dOm, kk * 2048), kIdescN128MN,
                      (t > 0 || kk > 0) ? 1u : 0u);
        }
        // the next tile's S^T over this tile's P^T (after the dV MMA in issue order)
        if (more) issue_s(dQn);
        // dK += dS^T Q_t: A from TMEM (dS^T over the dP^T columns)
        ok = mbar_wait(bar(B_DS), t & 1, abort_flag, prm.err, prm.wait_limit);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBQ / 16; ++kk) {
          const uint32_t acol = (kk >> 2) * 64 + (kk & 3) * 8;
          mma_bf16_ts(tmem + kTdK, tmem + kTP + acol, sdesc_add(dQm, kk * 2048), kIdescN128MN,
                      (t > 0 || kk > 0) ? 1u : 0u);
        }
        // both stages of tile t are free once dK is done (the compute
        // warpgroups read the tile's LSE and D before they released dS^T)
        tc_commit(bar(B_QE + sq));
        tc_commit(bar(B_OE + so));
        if (more) {
          ok = mbar_wait(bar(B_OF + so1), po1, abort_flag, prm.err, prm.wait_limit);
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
  } else {
    setmaxnreg_inc<kRegsComputeKV>();
    const int w = (warp - 4) >> 2, wq = warp & 3;  // w: query columns [64w, 64w + 64)
    const int row = wq * 32 + lane;                // key row within the tile
    const int j = n0 + row;
    int lo_j = 1, hi_j = 0;
    if (j < g.n) prm.mk.col_range(j, lo_j, hi_j);
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + kTS + 64 * w, tP = tmem + lane_off + kTP + 64 * w;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int e = t / nqt, i0 = (qt0 + t - e * nqt) * kBQ + 64 * w;  // this warpgroup's first query row
      const int sq = t % kQStages, so = t % kOStages;
      // LSE log2(e) and D of this warpgroup's 64 query rows (loaded with Q / dO)
      const float *lsm = reinterpret_cast<const float *>(smem + kOffLse + sq * kBQ * 4) + 64 * w;
      const float *dsm = reinterpret_cast<const float *>(smem + kOffD + so * kBQ * 4) + 64 * w;
      // phase a/b: P^T over this warpgroup's first 32 columns of S^T
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_QF + sq), (t / kQStages) & 1, abort_flag, prm.err, prm.wait_limit) &&
                                       mbar_wait(bar(B_SF), t & 1, abort_flag, prm.err, prm.wait_limit));
      if (!ok) break;
      tc_fence_after();
      const bool full = (i0 >= n0 + kBN - 1) && (i0 + 63 <= hi_a) && (i0 + 64 <= g.n) && (n0 + kBN <= g.n);
      uint32_t r[64];
      tmem_ld64(tS, r);
      // masked scores become -inf (exponential 0): the exponential loop has no branch
      if (!full) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (i0 + c < lo_j || i0 + c > hi_j) r[c] = __float_as_uint(-INFINITY);
      }
      uint32_t pp[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
#pragma unroll
        for (int u = 0; u < 2; ++u)
          r[c + u] = __float_as_uint(ex2_approx(fmaf(__uint_as_float(r[c + u]), prm.scale_log2, -lsm[c + u])));
        pp[c >> 1] = pack_bf16x2(__uint_as_float(r[c]), __uint_as_float(r[c + 1]));
      }
      tmem_st32_nowait(tS, pp);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_PS));
      // phase c: dS^T over this warpgroup's first 32 columns of dP^T
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OF + so), (t / kOStages) & 1, abort_flag, prm.err, prm.wait_limit) &&
                                       mbar_wait(bar(B_DPF), t & 1, abort_flag, prm.err, prm.wait_limit));
      if (!ok) break;
      tc_fence_after();
      uint32_t dp[64];
      tmem_ld64(tP, dp);
      uint32_t dd[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float d0 = __uint_as_float(r[c]) * (__uint_as_float(dp[c]) - dsm[c]);
        const float d1 = __uint_as_float(r[c + 1]) * (__uint_as_float(dp[c + 1]) - dsm[c + 1]);
        dd[c >> 1] = pack_bf16x2(d0, d1);
      }
      tmem_st32_nowait(tP, dd);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_DS));
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK (scaled)
    if (ok && T > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DONE), 0, abort_flag, prm.err, prm.wait_limit));
    tc_fence_after();
    __nv_bfloat16 *outp = (w == 0) ? prm.out0 : prm.out1;
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
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ================================================================== dQ
// One CTA = one 128-row query tile of one query head; Q and dO sit in TMEM
// as the A operands of S = Q K^T and dP = dO V^T over K/V tiles of 128 keys
// (all MMAs N=128).  The two compute warpgroups split each tile's key columns
// (64 each).  A tile is processed in two phases:
//   a. read S into registers (the S columns are then free and the next tile's
//      S is issued), P = exp2(S scale log2e - LSE log2e)
//   b. read dP, dS = P (dP - D), dS (bf16 pairs) over this warpgroup's own
//      dP columns -> dQ += dS K (A from TMEM), then the next tile's dP.
// TMEM: Q [0,64), dO [64,128) (bf16 pairs), dQ [128,256), S [256,384),
// dP / dS [384,512).  The next dP overwrites the dS the dQ MMA reads, which
// relies on tcgen05.mma executing in issue order.
namespace qk {
constexpr int kBM = 128;   // query rows per CTA
constexpr int kBK = 128;   // keys per K/V tile
constexpr int kStages = 3;
constexpr uint32_t kTile = 128 * 128 * 2;                  // one 128 x 128 bf16 tile
constexpr uint32_t kOffKV = 0;                             // stage s: K at 2s*kTile, V at (2s+1)*kTile
constexpr uint32_t kOffBar = kStages * 2 * kTile;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
constexpr uint32_t kTQ = 0, kTO = 64, kTdQ = 128, kTS = 256, kTP = 384;
}  // namespace qk

__global__ void __launch_bounds__(kThreads, 1)
    attn_dq_sm100_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const BwdParams prm) {
  using namespace qk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  enum { B_KF = 0, B_KE = kStages, B_SF = 2 * kStages, B_SR, B_DPF, B_DS, B_QO, B_DQ, B_DRAIN, B_N };
  static_assert(8 * B_N + 8 <= 256, "barrier area");
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffBar + 8 * B_N);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffBar + 8 * B_N + 4);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const HeadGeom &g = prm.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Blocks start in the order of their linear index (x fastest): with
  // kv_major the query tiles of one GQA group's heads at a time (the group's
  // heads side by side per tile), else those of every head side by side;
  // heaviest (latest) query tiles first either way.
  int rb, hh, mt;
  if (prm.kv_major) {
    const int nq = gridDim.y;
    const int lin = blockIdx.y * gridDim.x + blockIdx.x;
    const int unit = lin / (g.group * nq), rem = lin - unit * (g.group * nq);   // unit = (r*B + b)*gl + KV head
    mt = nq - 1 - rem / g.group;
    rb = unit / g.gl;
    hh = (unit - rb * g.gl) * g.group + rem % g.group;
  } else {
    const int qh = blockIdx.x;                   // (r*B + b)*hl + hh
    rb = qh / g.hl;
    hh = qh - rb * g.hl;
    mt = gridDim.y - 1 - blockIdx.y;
  }
  const int qh = rb * g.hl + hh;
  const int kvhead = rb * g.gl + hh / g.group;
  const int m0 = mt * kBM;

  int lo_first, hi_first, lo_last, hi_last;
  prm.mk.row_range(m0, lo_first, hi_first);
  prm.mk.row_range(min(m0 + kBM - 1, g.n - 1), lo_last, hi_last);
  const int jt0 = lo_first / kBK;
  const int NT = (hi_last >= lo_first) ? hi_last / kBK - jt0 + 1 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_N; ++i) mbar_init(bar(i), (i == B_SR || i == B_DS || i == B_QO) ? 256 : 1);
    *abort_flag = 0;
    fence_mbar_init();
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
  // Registers: producer / MMA warpgroup 120 per thread, the two compute
  // warpgroups 192 (a thread holds 64 columns of P and 64 of dP).

  if (warp < 4) {
    setmaxnreg_dec<kRegsCtlQ>();
    if (warp == 0) {
      if (lane == 0 && NT > 0) {
        int issued = 0;
        for (int j = 0; j < NT; ++j) {
          const int s = j % kStages, use = j / kStages;
          if (use > 0 && !mbar_wait(bar(B_KE + s), (use - 1) & 1, abort_flag, prm.err, prm.wait_limit)) break;
          const uint32_t st = sb + kOffKV + s * 2 * kTile;
          const int row0 = (jt0 + j) * kBK;
          mbar_arrive_expect_tx(bar(B_KF + s), 2 * kTile);
          for (int c = 0; c < 2; ++c) {
            tma_load_3d(st + c * 16384, &tmK, bar(B_KF + s), c * 64, row0, kvhead);
            tma_load_3d(st + kTile + c * 16384, &tmV, bar(B_KF + s), c * 64, row0, kvhead);
          }
          issued = j + 1;
        }
        // every copy issued lands before the CTA can exit
        for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
          mbar_wait(bar(B_KF + j % kStages), (j / kStages) & 1, nullptr, prm.err);
      }
    } else if (warp == 1) {
      if (lane == 0 && NT > 0) {
        bool ok = mbar_wait(bar(B_QO), 0, abort_flag, prm.err, prm.wait_limit);
        tc_fence_after();
        // S = Q K_j^T (A = Q from TMEM), dP = dO V_j^T (A = dO from TMEM); B tiles K-major
        auto issue_s = [&](uint64_t dK) {
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk)
            mma_bf16_ts(tmem + kTS, tmem + kTQ + kk * 8, sdesc_add(dK, (kk >> 2) * 16384 + (kk & 3) * 32),
                        kIdescN128, kk > 0);
          tc_commit(bar(B_SF));
        };
        auto issue_dp = [&](uint64_t dV) {
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk)
            mma_bf16_ts(tmem + kTP, tmem + kTO + kk * 8, sdesc_add(dV, (kk >> 2) * 16384 + (kk & 3) * 32),
                        kIdescN128, kk > 0);
          tc_commit(bar(B_DPF));
        };
        if (ok) ok = mbar_wait(bar(B_KF), 0, abort_flag, prm.err, prm.wait_limit);
        if (ok) {
          tc_fence_after();
          issue_s(sdesc_sw128(sb + kOffKV, 16, 1024));
          issue_dp(sdesc_sw128(sb + kOffKV + kTile, 16, 1024));
        }
        // Stages and parities roll forward; every descriptor of an iteration
        // is computed before its waits (nothing but MMAs right after a wait).
        int s = 0;
        uint32_t ps = 0;
        for (int j = 0; ok && j < NT; ++j) {
          const bool more = j + 1 < NT;
          const int s1 = (s + 1 == kStages) ? 0 : s + 1;
          const uint32_t ps1 = (s1 == 0) ? (ps ^ 1u) : ps;
          const uint32_t st = sb + kOffKV + s * 2 * kTile, st1 = sb + kOffKV + s1 * 2 * kTile;
          const uint64_t dKn = sdesc_sw128(st1, 16, 1024), dVn = sdesc_sw128(st1 + kTile, 16, 1024);
          const uint64_t dKm = sdesc_sw128(st, 16384, 1024);   // dQ: B = K tile, MN-major over d
          // both warpgroups hold S_j in registers, and the next K/V stage has
          // landed: the next tile's S (one wait point for both)
          ok = more ? mbar_wait2(bar(B_SR), j & 1, bar(B_KF + s1), ps1, abort_flag, prm.err, prm.wait_limit)
                    : mbar_wait(bar(B_SR), j & 1, abort_flag, prm.err, prm.wait_limit);
          if (!ok) break;
          tc_fence_after();
          if (more) issue_s(dKn);
          // dQ += dS K_j: A = dS from TMEM (key columns [0,64) in the dP
          // columns [0,32), [64,128) in [64,96))
          ok = mbar_wait(bar(B_DS), j & 1, abort_flag, prm.err, prm.wait_limit);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t acol = (kk >> 2) * 64 + (kk & 3) * 8;
            mma_bf16_ts(tmem + kTdQ, tmem + kTP + acol, sdesc_add(dKm, kk * 2048), kIdescN128MN,
                        (j > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar(B_KE + s));
          if (more) issue_dp(dVn);
          s = s1;
          ps = ps1;
        }
        if (ok) tc_commit(bar(B_DQ));
        // every MMA issued has completed before TMEM can be released
        tc_commit(bar(B_DRAIN));
        mbar_wait(bar(B_DRAIN), 0, nullptr, prm.err);
      }
    }
  } else {
    setmaxnreg_inc<kRegsComputeQ>();
    const int w = (warp - 4) >> 2, wq = warp & 3;   // w: key columns [64w, 64w + 64) of each tile
    const int row = wq * 32 + lane;
    const int i = m0 + row;
    const bool valid = i < g.n;
    int lo_i = 1, hi_i = 0;
    if (valid) prm.mk.row_range(i, lo_i, hi_i);
    const long long qrow = (long long)qh * g.n + i;
    const long long srow = (long long)qh * prm.n_pad + i;
    const float lse2 = valid ? prm.lse2[srow] : INFINITY;
    const float Di = valid ? prm.Dv[srow] : 0.f;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + kTS + 64 * w, tP = tmem + lane_off + kTP + 64 * w;
    // warpgroup 0 puts this row of Q into TMEM, warpgroup 1 the row of dO
    {
      const __nv_bfloat16 *src = (w == 0) ? prm.q : prm.dout;
      uint32_t v[64];
      const uint4 *p4 = reinterpret_cast<const uint4 *>(src + (valid ? qrow : 0) * kHD);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const uint4 w4 = valid ? __ldg(p4 + u) : make_uint4(0, 0, 0, 0);
        v[4 * u] = w4.x;
        v[4 * u + 1] = w4.y;
        v[4 * u + 2] = w4.z;
        v[4 * u + 3] = w4.w;
      }
      tmem_st64_nowait(tmem + lane_off + (w == 0 ? kTQ : kTO), v);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_QO));
    }
    bool ok = true;
    for (int j = 0; j < NT; ++j) {
      // phase a: P
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SF), j & 1, abort_flag, prm.err, prm.wait_limit));
      if (!ok) break;
      tc_fence_after();
      uint32_t r[64];
      tmem_ld64(tS, r);
      tc_fence_before();
      mbar_arrive(bar(B_SR));                  // the MMA thread may now overwrite S
      const int n0 = (jt0 + j) * kBK + 64 * w;
      const bool full = (n0 >= lo_last) && (n0 + 63 <= hi_first) && (n0 + 64 <= g.n);
      // masked scores become -inf (exponential 0): the exponential loop has no branch
      if (!full) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (n0 + c < lo_i || n0 + c > hi_i) r[c] = __float_as_uint(-INFINITY);
      }
#pragma unroll
      for (int c = 0; c < 64; ++c) r[c] = __float_as_uint(ex2_approx(fmaf(__uint_as_float(r[c]), prm.scale_log2, -lse2)));
      // phase b: dS over this warpgroup's first 32 columns of dP
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DPF), j & 1, abort_flag, prm.err, prm.wait_limit));
      if (!ok) break;
      tc_fence_after();
      uint32_t dp[64];
      tmem_ld64(tP, dp);
      uint32_t dd[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float d0 = __uint_as_float(r[c]) * (__uint_as_float(dp[c]) - Di);
        const float d1 = __uint_as_float(r[c + 1]) * (__uint_as_float(dp[c + 1]) - Di);
        dd[c >> 1] = pack_bf16x2(d0, d1);
      }
      tmem_st32_nowait(tP, dd);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_DS));
    }
    // epilogue: warpgroup w writes dQ columns [64w, 64w + 64)
    const long long orow = valid ? g.q_out_row(qh, i) : 0;
    if (ok && NT > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DQ), 0, abort_flag, prm.err, prm.wait_limit));
    tc_fence_after();
    if (ok && NT > 0) {
      uint32_t rr[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        tmem_ld32(tmem + lane_off + kTdQ + 64 * w + 32 * c, rr);
        if (valid) {
          uint4 *dptr = reinterpret_cast<uint4 *>(prm.out0 + orow * kHD + 64 * w + 32 * c);
          const float sc = g.scale;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 w4;
            w4.x = pack_bf16x2(__uint_as_float(rr[8 * u + 0]) * sc, __uint_as_float(rr[8 * u + 1]) * sc);
            w4.y = pack_bf16x2(__uint_as_float(rr[8 * u + 2]) * sc, __uint_as_float(rr[8 * u + 3]) * sc);
            w4.z = pack_bf16x2(__uint_as_float(rr[8 * u + 4]) * sc, __uint_as_float(rr[8 * u + 5]) * sc);
            w4.w = pack_bf16x2(__uint_as_float(rr[8 * u + 6]) * sc, __uint_as_float(rr[8 * u + 7]) * sc);
            dptr[u] = w4;
          }
        }
      }
    } else if (NT == 0 && valid) {
      uint4 *dptr = reinterpret_cast<uint4 *>(prm.out0 + orow * kHD + 64 * w);
      for (int u = 0; u < 8; ++u) dptr[u] = make_uint4(0, 0, 0, 0);
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

}  // namespace

uly_status attn_bf16_bwd_fused_launch(const HeadGeom &g, const MaskInfo &mk, const void *q, const void *k,
                                      const void *v, const void *dout, void *dq, void *dk, void *dv,
                                      const float *Dv, const float *L2, float *dq_acc, int n_pad,
                                      cudaStream_t stream);

// Workspace of the bf16 backward: D and LSE log2(e) (bwd_stats_stride floats
// each), then, for the fused backward, the fp32 dQ accumulator
// [query heads][n_pad][128] (256-byte aligned).
size_t attn_bf16_bwd_workspace(const HeadGeom &g, bool deterministic) {
  const long long rows_pad = (long long)g.P * g.B * g.hl * bwd_rows_padded(g.n);
  const size_t stats = 2 * sizeof(float) * (size_t)bwd_stats_stride(rows_pad);
  if (deterministic) return stats;
  return ((stats + 255) & ~size_t(255)) + (size_t)rows_pad * kHD * sizeof(float);
}

uly_status attn_bf16_bwd_launch(const uly_attn_desc *d, const HeadGeom &g, const MaskInfo &mk,
                                const void *q, const void *k, const void *v, const void *o,
                                const float *lse, const void *dout, void *dq, void *dk, void *dv,
                                float *workspace, cudaStream_t stream) {
  const int qheads = g.P * g.B * g.hl, kvheads = g.P * g.B * g.gl;
  const int n_pad = bwd_rows_padded(g.n);
  const long long rows_pad = (long long)qheads * n_pad;
  const bool fused = d->deterministic == 0;
  float *Dv = workspace;
  float *L2 = workspace + bwd_stats_stride(rows_pad);
  float *dq_acc = nullptr;
  if (fused) {
    const size_t stats = 2 * sizeof(float) * (size_t)bwd_stats_stride(rows_pad);
    dq_acc = reinterpret_cast<float *>(reinterpret_cast<char *>(workspace) + ((stats + 255) & ~size_t(255)));
  }
  if (rows_pad > 0) {
    prof::Scope scope(prof::K_ATTN_BWD_STATS, stream);
    attn_bwd_stats_kernel<<<(unsigned)((rows_pad + 15) / 16), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(dout), lse, Dv, L2, dq_acc,
        g, n_pad, rows_pad);
    note_launches(1);
  }
  if (fused)
    return attn_bf16_bwd_fused_launch(g, mk, q, k, v, dout, dq, dk, dv, Dv, L2, dq_acc, n_pad, stream);
  CUtensorMap mK128, mV128, mQ128, mO128, mK64, mV64;
  if (!make_tmap_heads_bf16(&mK128, k, kHD, g.n, kvheads, 128) ||
      !make_tmap_heads_bf16(&mV128, v, kHD, g.n, kvheads, 128) ||
      !make_tmap_heads_bf16(&mQ128, q, kHD, g.n, qheads, 128) ||
      !make_tmap_heads_bf16(&mO128, dout, kHD, g.n, qheads, 128) ||
      !make_tmap_heads_bf16(&mK64, k, kHD, g.n, kvheads, 64) ||
      !make_tmap_heads_bf16(&mV64, v, kHD, g.n, kvheads, 64))
    return ULY_ERR_CUDA;
  static std::atomic<uint64_t> optin_kv{0}, optin_q{0};
  if (!smem_optin(attn_dkdv_sm100_kernel, kv::kSmemBytes, optin_kv) ||
      !smem_optin(attn_dq_sm100_kernel, qk::kSmemBytes, optin_q))
    return ULY_ERR_CUDA;
  BwdParams prm;
  prm.q = static_cast<const __nv_bfloat16 *>(q);
  prm.dout = static_cast<const __nv_bfloat16 *>(dout);
  prm.lse2 = L2;
  prm.Dv = Dv;
  prm.n_pad = n_pad;
  prm.g = g;
  prm.mk = mk;
  prm.scale_log2 = g.scale * kLog2e;
  prm.err = error_word();
  prm.wait_limit = wait_limit_cycles();
  prm.out0 = static_cast<__nv_bfloat16 *>(dv);
  prm.out1 = static_cast<__nv_bfloat16 *>(dk);
  dim3 gkv(kvheads, (g.n + kv::kBN - 1) / kv::kBN);
  prm.kv_major = attn_kv_head_major(mk.mask, gkv.y) ? 1 : 0;
  {
    prof::Scope scope(prof::K_ATTN_DKDV_SM100, stream);
    attn_dkdv_sm100_kernel<<<gkv, kThreads, kv::kSmemBytes, stream>>>(mK128, mV128, mQ128, mO128, prm);
  }
  prm.out0 = static_cast<__nv_bfloat16 *>(dq);
  prm.out1 = nullptr;
  dim3 gq(qheads, (g.n + qk::kBM - 1) / qk::kBM);
  prm.kv_major = attn_kv_head_major(mk.mask, (long long)gq.y * g.group) ? 1 : 0;
  {
    prof::Scope scope(prof::K_ATTN_DQ_SM100, stream);
    attn_dq_sm100_kernel<<<gq, kThreads, qk::kSmemBytes, stream>>>(mK128, mV128, prm);
  }
  note_launches(2);
  return last_launch_status();
}

}  // namespace uly
