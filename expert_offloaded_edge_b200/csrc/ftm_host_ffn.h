// Host-side expert FFN of the bandwidth-adaptive miss split (internal).
#pragma once
#include <cstddef>
#include <cstdint>

#include "ftm.h"

namespace ftm {

// One expert's rows for the host FFN: the expert's bank in host memory and one
// pointer per row to its input activation and to its output row (bf16, fp32
// for FTM_F32 layers, d elements each).
struct HostGroup {
  const uint8_t* bank;
  int n;
  const uint8_t* const* x;
  uint8_t* const* y;
};

// fp32 scratch the host FFN needs for `rows` rows in all.
size_t host_ffn_scratch_bytes(const ftm_layer_desc* L, int64_t rows);
// 1 if the host FFN handles this weight dtype (every ftm_wdtype).
int host_ffn_supported(int wdtype);
// threads > 0, else the hardware thread count.
int host_threads(int threads);
// act_scale: host fp32[2], the NVFP4 activation global scales {gx, gh}, or NULL (1, 1).
void host_ffn_groups(const ftm_layer_desc* L, const ftm_bank_layout* bl, const HostGroup* groups, int ng,
                     const float* act_scale, float* scratch, int threads);

}  // namespace ftm
