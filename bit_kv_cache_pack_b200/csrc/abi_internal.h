// Host-side helpers shared by the C-ABI entry points (internal).
#pragma once

#include <stdint.h>

#include "../../include/omnikv.h"
#include "kernels.h"

namespace omnikv {

// The split count num_splits resolves to (0 = library default).
int32_t resolve_splits(const omnikv_config* cfg, const omnikv_cache* c, int32_t requested);

// Validate arguments and fill the launch parameters; nothing is launched.
omnikv_status prepare_decode(const omnikv_config* cfg, const omnikv_cache* cache, const void* q, void* partials,
                             int32_t num_splits, DecodeParams* p);
omnikv_status prepare_combine(const omnikv_config* cfg, const omnikv_cache* cache, const void* partials,
                              int32_t num_splits, float* out, CombineParams* p);
omnikv_status validate_config_cache(const omnikv_config* cfg, const omnikv_cache* cache);

}  // namespace omnikv
