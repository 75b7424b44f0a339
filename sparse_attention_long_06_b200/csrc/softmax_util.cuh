// Cross-thread reductions used by the softmax warpgroups (128 threads, four
// warps, one TMEM lane quadrant each).
#pragma once
#include <cstdint>

namespace nsa {

template <int kBarrier>
__device__ __forceinline__ void named_bar_128() {
  asm volatile("bar.sync %0, 128;" ::"n"(kBarrier) : "memory");
}

// Max (is_max) or sum of 16 per-thread values over the 128 threads of a
// warpgroup.  A reduce-scatter butterfly (16 shuffles) leaves lane pair
// (2j, 2j+1) of each warp with column col(lane) of its warp; the four warp
// partials meet in shared memory laid out [column][warp] (`red`, 64 floats,
// 16-byte aligned), and every thread reads back all 16 columns.  Uses named
// barrier kBarrier once.
template <int kBarrier>
__device__ __forceinline__ void reduce16_across_128(float (&v)[16], float* red, int q4, int lane,
                                                    bool is_max) {
  float a[8];
  {
    const bool up = lane & 16;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float send = up ? v[j] : v[j + 8];
      const float keep = up ? v[j + 8] : v[j];
      const float r = __shfl_xor_sync(0xffffffffu, send, 16);
      a[j] = is_max ? fmaxf(keep, r) : keep + r;
    }
  }
#pragma unroll
  for (int o = 8, half = 4; o >= 2; o >>= 1, half >>= 1) {
    const bool up = lane & o;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (j < half) {
        const float send = up ? a[j] : a[j + half];
        const float keep = up ? a[j + half] : a[j];
        const float r = __shfl_xor_sync(0xffffffffu, send, o);
        a[j] = is_max ? fmaxf(keep, r) : keep + r;
      }
    }
  }
  {
    const float r = __shfl_xor_sync(0xffffffffu, a[0], 1);
    a[0] = is_max ? fmaxf(a[0], r) : a[0] + r;
  }
  const int col = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
                  ((lane >> 1) & 1);
  if ((lane & 1) == 0) red[col * 4 + q4] = a[0];
  named_bar_128<kBarrier>();
#pragma unroll
  for (int h = 0; h < 16; ++h) {
    const float4 p = *reinterpret_cast<const float4*>(red + h * 4);
    v[h] = is_max ? fmaxf(fmaxf(p.x, p.y), fmaxf(p.z, p.w)) : (p.x + p.y) + (p.z + p.w);
  }
}

}  // namespace nsa
