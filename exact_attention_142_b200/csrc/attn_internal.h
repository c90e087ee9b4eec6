// attn_internal.h -- declarations shared by the library's translation units
// (not part of the C ABI).
#pragma once

namespace attn {
// Read and clear the decode kernels' device status word; returns ATTN_OK or
// ATTN_ERR_CUDA.
int decode_status_take(int* value);
// The same for the backward kernels.
int bwd_status_take(int* value);
}  // namespace attn
