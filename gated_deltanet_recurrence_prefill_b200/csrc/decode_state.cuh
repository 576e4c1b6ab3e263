// decode_state.cuh -- loads and stores of 4 consecutive state elements of a
// row (lane `lane` of the row's 32), for a float32 state or a bf16 one.  The
// state is streamed once per step, so both use the evict-first cache hints.
#pragma once

#include "common.cuh"

namespace gdn {

GDN_DEVICE float4 state_load4(const float* row, int lane) {
    return __ldcs(reinterpret_cast<const float4*>(row) + lane);
}
GDN_DEVICE void state_store4(float* row, int lane, float4 v) {
    __stcs(reinterpret_cast<float4*>(row) + lane, v);
}

// bf16 state: 8 bytes per lane; rounded to nearest even when stored
GDN_DEVICE float4 state_load4(const uint16_t* row, int lane) {
    const uint2 r = __ldcs(reinterpret_cast<const uint2*>(row) + lane);
    const float2 a = bf16x2_to_f32x2(r.x), b = bf16x2_to_f32x2(r.y);
    return make_float4(a.x, a.y, b.x, b.y);
}
GDN_DEVICE void state_store4(uint16_t* row, int lane, float4 v) {
    __stcs(reinterpret_cast<uint2*>(row) + lane, make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w)));
}

}  // namespace gdn
