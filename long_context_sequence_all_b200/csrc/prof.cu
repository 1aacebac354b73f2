// Per-kernel CUDA-event timing (see prof.cuh) and its C ABI.
#include <mutex>
#include <vector>

#include "common.cuh"
#include "prof.cuh"

namespace uly {
namespace prof {

namespace {

struct Pending {
  int kernel;
  cudaEvent_t start, stop;
  bool closed;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Pending> g_pending;        // events recorded since the last read
std::vector<cudaEvent_t> g_free;       // reusable events
double g_ms[K_COUNT] = {0};
long long g_count[K_COUNT] = {0};

cudaEvent_t take_event() {
  if (!g_free.empty()) {
    cudaEvent_t e = g_free.back();
    g_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

const char *name(int k) {
  static const char *names[K_COUNT] = {
      "seq_to_head", "head_to_seq", "loss_partial", "loss_finalize", "attn_fwd_f32",
      "attn_dq_f32", "attn_dkdv_f32", "attn_bwd_dot", "attn_fwd_sm100", "attn_dkdv_sm100",
      "attn_dq_sm100", "attn_bwd_stats", "loss_fwd_bwd", "kv_seq_to_head_rep",
      "kv_head_to_seq_sum", "shift_labels", "rope_table", "qkv_proj_sm100",
      "o_proj_sm100", "check_cu_seqlens", "attn_bwd_sm100", "attn_dq_convert",
      "seq_to_head_vec", "head_to_seq_vec", "qkv_dy", "qkv_proj_dx_sm100", "qkv_proj_dw_sm100",
      "o_proj_do_sm100", "o_proj_dw_sm100"};
  return (k >= 0 && k < K_COUNT) ? names[k] : "unknown";
}

bool enabled() { return g_on; }

Scope::Scope(int kernel, cudaStream_t stream) : kernel_(kernel), stream_(stream), slot_(-1) {
  if (!g_on) return;
  std::lock_guard<std::mutex> lk(g_mu);
  cudaEvent_t a = take_event(), b = take_event();
  if (!a || !b) return;
  if (cudaEventRecord(a, stream_) != cudaSuccess) return;
  g_pending.push_back({kernel_, a, b, false});
  slot_ = (int)g_pending.size() - 1;
}

void Scope::end() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (slot_ < (int)g_pending.size() && !g_pending[slot_].closed) {
    cudaEventRecord(g_pending[slot_].stop, stream_);
    g_pending[slot_].closed = true;
  }
  slot_ = -1;
}

// Fold every closed pending pair into the totals (waits for the events).
void drain() {
  std::lock_guard<std::mutex> lk(g_mu);
  for (Pending &p : g_pending) {
    if (p.closed && cudaEventSynchronize(p.stop) == cudaSuccess) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, p.start, p.stop) == cudaSuccess) {
        g_ms[p.kernel] += ms;
        g_count[p.kernel] += 1;
      }
    }
    g_free.push_back(p.start);
    g_free.push_back(p.stop);
  }
  g_pending.clear();
}

void reset_totals() {
  std::lock_guard<std::mutex> lk(g_mu);
  for (int k = 0; k < K_COUNT; ++k) {
    g_ms[k] = 0;
    g_count[k] = 0;
  }
}

void set_on(bool on) { g_on = on; }

void totals(int k, double *ms, long long *count) {
  std::lock_guard<std::mutex> lk(g_mu);
  *ms = g_ms[k];
  *count = g_count[k];
}

}  // namespace prof
}  // namespace uly

using namespace uly;

extern "C" {

uly_status ulysses_profile_enable(int32_t on) {
  prof::drain();
  prof::reset_totals();
  prof::set_on(on != 0);
  return ULY_OK;
}

uly_status ulysses_profile_read(int32_t kernel, double *total_ms, int64_t *launches) {
  if (!total_ms || !launches) return ULY_ERR_NULL;
  if (kernel < 0 || kernel >= prof::K_COUNT) return ULY_ERR_SHAPE;
  prof::drain();
  long long c = 0;
  prof::totals(kernel, total_ms, &c);
  *launches = c;
  return ULY_OK;
}

const char *ulysses_kernel_name(int32_t kernel) { return prof::name(kernel); }

int32_t ulysses_kernel_count(void) { return prof::K_COUNT; }

}  // extern "C"
