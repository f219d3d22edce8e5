// Functions shared between the library's translation units but not exported
// (hidden visibility: they are not part of the C ABI in include/tpblock.h).
#pragma once

#define TP_INTERNAL __attribute__((visibility("hidden")))

// The argument checks tp_mlp_forward makes before anything else (pointers,
// alignment, enums, eps, shapes).  Returns TP_OK or the status that
// tp_mlp_forward would return for these arguments.
TP_INTERNAL int tp_internal_check_mlp_args(int S, int H, int F, int t, int dtype, int out_dtype, const void* X,
                                           const void* const* A_shards, const void* const* B_shards,
                                           const float* gamma, const float* beta, float eps, int act,
                                           const void* Y);
