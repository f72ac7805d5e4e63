// simt.cuh -- small CUDA-core helpers shared by the kernels: paired fp32
// fused multiply-add and add, and a transposed reduction of several values
// over a group of lanes.
#pragma once

namespace sattn {

// d = a0 * b0 + c0, d1 = a1 * b1 + c1 as one paired fp32 instruction
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                     float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// d0 += a0, d1 += a1 as one paired fp32 instruction
__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1) {
  asm("{\n\t.reg .b64 ra, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rd, {%0, %1};\n\t"
      "add.rn.f32x2 rd, rd, ra;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1));
}

// Sum NV per-lane values over each group of W consecutive lanes (W a power
// of two, `mask` the lanes taking part), transposed: each level hands half of
// the remaining values to the partner lane, so the reduction costs
// NV - 1 + log2(W / NV) shuffles (NV <= W) instead of NV log2(W).
// Afterwards lane l of a group (sub = l % W) holds max(1, NV / W) sums in
// v[0..]: value index sub / (W / NV) when NV <= W, sub * (NV / W) + q
// otherwise.
template <int NV, int W>
__device__ __forceinline__ void group_reduce_transposed(float (&v)[NV], unsigned mask, int lane) {
  int nv = NV;
#pragma unroll
  for (int o = W / 2; o >= 1; o >>= 1) {
    if (nv > 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int q = 0; q < NV / 2; ++q) {
        if (q < nv / 2) {
          const float send = upper ? v[q] : v[q + nv / 2];
          const float keep = upper ? v[q + nv / 2] : v[q];
          v[q] = keep + __shfl_xor_sync(mask, send, o);
        }
      }
      nv >>= 1;
    } else {
      v[0] += __shfl_xor_sync(mask, v[0], o);
    }
  }
}

}  // namespace sattn
