// moe_paths.cuh -- the fused whole-layer forward (layer.cu).
#pragma once
#include "moe_internal.cuh"

namespace moe {
size_t layer_ws_bytes(const moe_layer_args &a);
moe_status layer_forward(const moe_layer_args &a, void *ws, size_t ws_bytes, cudaStream_t s);
}  // namespace moe
