// seg_stream.cu -- the carried state of segmented execution, one segment at
// a time.
//
// "Training-Inference Consistent Segmented Execution for Long-Context LLMs"
// (section 整体框架): the layer is an operator applied per segment,
// (C_i, o^(i)) = F(x^(i), C_{i-1}, R_{i-1}), where C_{i-1} is what the local
// heads carry (the tail of the previous tokens) and R_{i-1} what the long
// heads retrieve from (the read-only pool of earlier keys, scored with the
// previous segment's last query).  The state buffer holds exactly that:
// every earlier token's raw K and V (the pool, and the tail's source), their
// keys rotated at their global positions (the band the attention kernel
// reads), the previous segment's last query of every head, and a header
// counting the segments taken.  A step appends its segment and replaces the
// query; the attention, retrieval and rotation kernels are the whole-layer
// ones, pointed at the state.
//
//   segstate_reset_kernel   writes the header (no segment taken yet);
//   segstate_append_kernel  checks that the step is the next segment (else
//                           the status word gets SATTN_ERR_INVALID_ARG and
//                           nothing of the state is written) and copies the
//                           segment's raw K and V rows into the history;
//   segstate_finish_kernel  the segment's last query of every head replaces
//                           the carried one; the header counts the segment.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "status.cuh"

namespace sattn {

namespace {

constexpr int32_t kStateMagic = 0x53454753;  // "SEGS"

__global__ void segstate_reset_kernel(int32_t* header, int S, int T_cap) {
  if (threadIdx.x == 0) {
    header[0] = kStateMagic;
    header[1] = 0;  // segments taken
    header[2] = S;
    header[3] = T_cap;
  }
}

// the step is segment `seg` of a state configured for (S, T_cap)
__device__ __forceinline__ bool step_ok(const SegStateArgs& a) {
  const volatile int32_t* h = a.header;
  return h[0] == kStateMagic && h[1] == a.seg && h[2] == a.S && h[3] == a.T_cap;
}

// grid-stride over 16-byte pieces of the segment's K and V rows
__global__ void segstate_append_kernel(SegStateArgs a) {
  const bool ok = step_ok(a);
  if (!ok) {
    if (blockIdx.x == 0 && threadIdx.x == 0 && atomicCAS(a.status, 0, SATTN_ERR_INVALID_ARG) == 0)
      atomicExch(a.status + 1, 90);
    return;
  }
  const int pieces = a.d / 8;  // 16-byte pieces per row
  const int64_t n = (int64_t)a.B * a.Hkv * a.S * pieces;
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n; x += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(x % pieces);
    int64_t r = x / pieces;
    const int t = (int)(r % a.S);
    r /= a.S;
    const int h = (int)(r % a.Hkv);
    const int b = (int)(r / a.Hkv);
    const int64_t dst = (((int64_t)b * a.Hkv + h) * a.T_cap + (int64_t)a.seg * a.S + t) * a.d + c * 8;
    const uint4 kv = *reinterpret_cast<const uint4*>(a.K + b * a.k_sb + h * a.k_sh + t * a.k_st + c * 8);
    const uint4 vv = *reinterpret_cast<const uint4*>(a.V + b * a.v_sb + h * a.v_sh + t * a.v_st + c * 8);
    *reinterpret_cast<uint4*>(a.Khist + dst) = kv;
    *reinterpret_cast<uint4*>(a.Vhist + dst) = vv;
  }
}

// grid (B * Hq): one block per (batch, head)
__global__ void segstate_finish_kernel(SegStateArgs a) {
  if (status_failed(a.status)) return;
  const int bh = blockIdx.x;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const __nv_bfloat16* q = a.Q + b * a.q_sb + h * a.q_sh + (int64_t)(a.S - 1) * a.q_st;
  __nv_bfloat16* dst = a.q_end + (int64_t)bh * a.d;
  for (int c = threadIdx.x; c < a.d; c += blockDim.x) dst[c] = q[c];
  // every block has read the header before the append kernel ended, so
  // counting the segment here cannot be seen by this step's checks
  if (bh == 0 && threadIdx.x == 0) a.header[1] = a.seg + 1;
}

}  // namespace

cudaError_t launch_segstate_reset(int32_t* header, int S, int T_cap, cudaStream_t st) {
  segstate_reset_kernel<<<1, 32, 0, st>>>(header, S, T_cap);
  return cudaGetLastError();
}

cudaError_t launch_segstate_append(const SegStateArgs& a, cudaStream_t st) {
  const int64_t n = (int64_t)a.B * a.Hkv * a.S * (a.d / 8);
  const int64_t want = (n + 255) / 256;
  const int64_t cap = (int64_t)sm_count() * 8;
  segstate_append_kernel<<<(unsigned)(want < cap ? (want > 0 ? want : 1) : cap), 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_segstate_finish(const SegStateArgs& a, cudaStream_t st) {
  segstate_finish_kernel<<<(unsigned)(a.B * a.Hq), 128, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace sattn
