// Opt-in per-kernel timing: when enabled (ulysses_profile_enable), every
// kernel launch of the library is bracketed by two CUDA events recorded on
// the launch's own stream; ulysses_profile_read() waits for them and reports
// the summed device time and launch count per kernel.  Disabled, it costs one
// branch per launch.
#pragma once

#include <cuda_runtime.h>

namespace uly {
namespace prof {

enum Kernel {
  K_SEQ_TO_HEAD = 0,
  K_HEAD_TO_SEQ,
  K_LOSS_PARTIAL,
  K_LOSS_FINALIZE,
  K_ATTN_FWD_F32,
  K_ATTN_DQ_F32,
  K_ATTN_DKDV_F32,
  K_ATTN_BWD_DOT,
  K_ATTN_FWD_SM100,
  K_ATTN_DKDV_SM100,
  K_ATTN_DQ_SM100,
  K_ATTN_BWD_STATS,
  K_LOSS_FWD_BWD,
  K_KV_REPLICATE,
  K_KV_REDUCE,
  K_SHIFT_LABELS,
  K_ROPE_TABLE,
  K_QKV_PROJ,
  K_O_PROJ,
  K_CHECK_CU,
  K_ATTN_BWD_SM100,
  K_ATTN_DQ_CONVERT,
  K_SEQ_TO_HEAD_VEC,
  K_HEAD_TO_SEQ_VEC,
  K_QKV_DY,
  K_QKV_DX,
  K_QKV_DW,
  K_O_PROJ_DO,
  K_O_PROJ_DWO,
  K_COUNT
};

const char *name(int k);
bool enabled();
// Records the start event (if enabled) in the constructor and the end event
// in end() / the destructor.
class Scope {
 public:
  Scope(int kernel, cudaStream_t stream);
  ~Scope() { end(); }
  void end();

 private:
  int kernel_;
  cudaStream_t stream_;
  int slot_;
};

}  // namespace prof
}  // namespace uly
