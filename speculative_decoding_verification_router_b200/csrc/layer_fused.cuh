// The fused verify-layer kernel's host interface (layer_fused.cu), used by
// the whole-layer entry point (api.cu).
#pragma once

#include "ms_common.cuh"

namespace ms {

// Device buffers of one fused-layer launch, all inside the layer workspace.
struct LfBuffers {
    __nv_bfloat16 *x_pad, *x_perm, *h_perm, *h_sh;   // the expert workspace's token operands and activations
    float* partials;                                  // split-tile partial sums
    float *logits, *y_perm, *y_sh;                    // [T][E] router logits, [T*k][H] and [T][H] expert outputs
    int32_t *idx, *off, *perm, *slot;                 // the routing, as the stand-alone calls would write it
    float* w;
    int32_t* status;                                  // device status word
    unsigned int* bar;                                // grid-barrier counter (zeroed with the status word)
    int rows_pad, t_pad;                              // rows of x_perm / h_perm and of h_shared
};

// Whether one fused launch covers a layer of this shape on the current device.
bool layer_fused_supported(int T, int H, int E, int I, int S, int k);
ms_status layer_fused_launch(const float* a, const float* wr, const float* bias, const void* wgu, const void* wd,
                             const void* wsgu, const void* wsd, int T, int H, int E, int I, int S, int k, int renorm,
                             float eps, float* out, const LfBuffers& b, cudaStream_t s);
// The expert workspace's token operands, activations and partial sums (expert_ffn.cu).
void ffn_ws_buffers(void* ws, int T, int H, int E, int I, int S, int k, LfBuffers& b);

}  // namespace ms
