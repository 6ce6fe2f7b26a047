// capi_internal.h -- argument checks and parameter builders of the C ABI
// (capi.cu) shared with the library's other entry-point files, so that
// every entry point that takes a layout accepts and refuses the same
// inputs.  Internal to libmoe_layout.so.
#pragma once

#include "moe_kernels.h"
#include "moe_layout.h"

namespace moe {

// MOE_OK, or MOE_ERR_INVALID_ARG when an array the configuration needs is
// NULL (per-token arrays may be NULL only when there are no tokens).
moe_status_t check_layout_ptrs(const moe_config_t* c, const moe_layout_t* L);

// The layout launcher's parameters for cfg / topk_idx / L (L->workspace is
// taken as the scratch; callers with other scratch overwrite it).
LayoutParams layout_params(const moe_config_t* c, const int32_t* topk_idx, const moe_layout_t* L);

}  // namespace moe
