// internal.h -- entry points shared between the library's own translation units.
#pragma once

#include <cstddef>
#include <cstdint>

#include "mlora.h"

// mlora_apply with the long-segment H workspace in caller-provided device memory of
// `ws_bytes` bytes; never allocates.  MLORA_ERR_UNSUPPORTED if the batch needs more.
mlora_status mlora_apply_with_workspace(mlora_pool *pool, const mlora_segments *segs,
                                        const void *X, int64_t ldx, void *Y, int64_t ldy,
                                        void *stream, float *ws, size_t ws_bytes);

// Look up (and so reserve, under lazy module loading) the no-allocation entry point's
// scratch array on device `dev`, which must be current; cached per device.
mlora_status mlora_noalloc_reserve(int dev);

// Device the pool was created on (-1 for NULL).
int mlora_pool_device(const mlora_pool *pool);
