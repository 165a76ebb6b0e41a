// Fine-grained M x 1 key-slice path: group-mean queries, exact per-head
// threshold, slice bitmask, and gather attention over the kept keys.
#include "sa_fg.h"

namespace sa {

size_t fg_qbar_bytes(int BH, int G, int d) { return sizeof(float) * (size_t)BH * G * d; }
size_t fg_hist_bytes(int BH) { return sizeof(uint32_t) * (size_t)BH * 4096; }
size_t fg_sel_bytes(int BH) { return sizeof(uint32_t) * (size_t)BH * 8; }

cudaError_t launch_fg_build(const FgBuildParams&, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_fg_attn(const FgAttnParams&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace sa
