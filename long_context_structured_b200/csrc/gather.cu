// gather.cu -- K3: separator K/V gather.
//
// SepLLM ("SepLLM", CSDN article, sections 五.2 and 6.2) keeps every earlier
// separator token; their keys and values are scattered through the
// sequence.  This pass copies them, in the compacted order of the block map,
// into dense per-(batch, kv-head) arrays so the attention kernel can stream
// them as ordinary 128-row tiles through the tensor-memory-access engine.
// Rows between the separator count and the next multiple of 128 are zeroed
// (they are masked, and zero keeps the masked products finite).
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace sattn {

namespace {

// grid (Tpad/128, Hkv, B), 256 threads: 8 warps x 16 rows
__global__ void sep_gather_kernel(GatherArgs a) {
  const int b = blockIdx.z, g = blockIdx.y;
  const int count = a.sep_count[b];
  const int padded = (count + kTile - 1) / kTile * kTile;
  const int r_base = blockIdx.x * kTile;
  if (r_base >= padded) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vec = a.d / 8;  // 16-byte vectors per row (16 for d = 128)
  __nv_bfloat16* kd = a.Ks + ((size_t)b * a.Hkv + g) * a.Tpad * a.d;
  __nv_bfloat16* vd = a.Vs + ((size_t)b * a.Hkv + g) * a.Tpad * a.d;
  for (int rr = warp; rr < kTile; rr += 8) {
    const int r = r_base + rr;
    // lanes 0..vec-1 copy K, lanes 16..16+vec-1 copy V
    const int part = lane >> 4, x = lane & 15;
    if (x >= vec) continue;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < count) {
      const int j = a.sep_pos[(size_t)b * a.T + r];
      const __nv_bfloat16* src = part == 0 ? a.Ksrc + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st
                                           : a.Vsrc + b * a.v_sb + g * a.v_sh + (int64_t)j * a.v_st;
      val = reinterpret_cast<const uint4*>(src)[x];
    }
    __nv_bfloat16* dst = (part == 0 ? kd : vd) + (size_t)r * a.d;
    reinterpret_cast<uint4*>(dst)[x] = val;
  }
}

}  // namespace

cudaError_t launch_sep_gather(const GatherArgs& a, cudaStream_t st) {
  if (a.B == 0 || a.Hkv == 0 || a.Tpad == 0) return cudaSuccess;
  dim3 grid(a.Tpad / kTile, a.Hkv, a.B);
  sep_gather_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace sattn
