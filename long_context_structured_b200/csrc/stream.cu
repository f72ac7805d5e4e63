// stream.cu -- SepLLM's streaming KV cache for generation ("SepLLM", section
// 6.2): an Initial cache (a slots), a Separator cache (s slots), a Local
// window (w slots) and a Past window that takes what overflows the local
// one.  When the running size reaches the capacity c, the separators in Past
// move to the Separator cache (the oldest separators go if more than s would
// stay) and the rest of Past is dropped.  The slots are ordered Initial |
// Separator | Past | Local with the newest token last, so a decoding step is
// attention over the first size slots with rolled positions (the talk page,
// section "Streaming ARMS": key x at rotary position x).
//
// State (caller-owned device memory, laid out by stream_layout()): per
// sequence the four region sizes, the cache length, a compaction plan, the
// stream position and separator flag of every slot, K and V [B, Hkv, c, d]
// and a scratch copy of the same shape for compaction.  Every decision is
// taken on the device, so an append is four launches with no host round
// trip:
//   stream_append_kernel   the new token's K, V row into the slot after the
//                          last one (the cache always has room: after each
//                          append the size is below c);
//   stream_plan_kernel     one block per sequence: region sizes; when the
//                          size reaches c, the destination of every slot
//                          (block-wide prefix count of Past's separators);
//   stream_move_kernel     (twice) kept rows to their new slots through the
//                          scratch copy (sources and destinations overlap).
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace sattn {

namespace {

constexpr int kPlanThreads = 256;

// one block per (b, g); d/8 threads, each copying 16 bytes of K and of V
__global__ void stream_append_kernel(StreamArgs a) {
  const int bg = blockIdx.x;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int slot = a.len[b];
  const int x = threadIdx.x;
  const size_t src = ((size_t)b * a.Hkv + g) * a.d + x * 8;
  const size_t dst = (((size_t)b * a.Hkv + g) * a.c + slot) * a.d + x * 8;
  *reinterpret_cast<uint4*>(a.K + dst) = *reinterpret_cast<const uint4*>(a.K_new + src);
  *reinterpret_cast<uint4*>(a.V + dst) = *reinterpret_cast<const uint4*>(a.V_new + src);
  if (g == 0 && x == 0) {
    a.pos[(size_t)b * a.c + slot] = (int32_t)a.position;
    a.flag[(size_t)b * a.c + slot] = a.sep_new ? (a.sep_new[b] ? 1 : 0) : 0;
  }
}

// one block per sequence
__global__ void __launch_bounds__(kPlanThreads) stream_plan_kernel(StreamArgs a) {
  __shared__ int warp_tot[kPlanThreads / 32];
  __shared__ int carry;
  const int b = blockIdx.x;
  int32_t* sz = a.sizes + 4 * b;
  int n_init = sz[0], n_sep = sz[1], n_past = sz[2], n_local = sz[3];
  // the appended token: Initial while the stream is in its first a tokens,
  // else the Local window, whose oldest entry moves to Past beyond w
  if (n_init < a.a && n_sep == 0 && n_past == 0 && n_local == 0) {
    ++n_init;
  } else {
    ++n_local;
    if (n_local > a.w) {
      --n_local;
      ++n_past;
    }
  }
  const int total = n_init + n_sep + n_past + n_local;
  __syncthreads();  // every thread has read the old sizes
  if (total < a.c) {
    if (threadIdx.x == 0) {
      sz[0] = n_init;
      sz[1] = n_sep;
      sz[2] = n_past;
      sz[3] = n_local;
      a.len[b] = total;
      a.ctrl[2 * b] = 0;
    }
    return;
  }
  // compaction: separators of Past after the cached ones, oldest dropped beyond s
  const int S0 = n_init, S1 = S0 + n_sep, P1 = S1 + n_past;
  const uint8_t* fl = a.flag + (size_t)b * a.c;
  int32_t* dst = a.dst + (size_t)b * a.c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  // pass 1: count Past's separators
  int cnt = 0;
  for (int k = S1 + threadIdx.x; k < P1; k += kPlanThreads) cnt += fl[k] ? 1 : 0;
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) warp_tot[warp] = cnt;
  __syncthreads();
  int n_new = 0;
  for (int w = 0; w < kPlanThreads / 32; ++w) n_new += warp_tot[w];
  const int all_sep = n_sep + n_new;
  const int drop = all_sep > a.s ? all_sep - a.s : 0;
  const int n_sep2 = all_sep - drop;
  // pass 2: destinations; Past's separators need their rank (exclusive prefix count)
  for (int k = threadIdx.x; k < S1; k += kPlanThreads) {
    if (k < S0) dst[k] = k;
    else dst[k] = (k - S0 < drop) ? -1 : S0 + (k - S0) - drop;
  }
  for (int k = P1 + threadIdx.x; k < total; k += kPlanThreads) dst[k] = S0 + n_sep2 + (k - P1);
  for (int base = S1; base < P1; base += kPlanThreads) {
    const int k = base + threadIdx.x;
    const int f = (k < P1 && fl[k]) ? 1 : 0;
    int incl = f;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    __syncthreads();  // warp_tot of the previous round is consumed
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = carry;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    if (k < P1) {
      const int rank = n_sep + before + incl - f;  // among all separators, old first
      dst[k] = f ? ((rank < drop) ? -1 : S0 + rank - drop) : -1;
    }
    __syncthreads();
    if (threadIdx.x == kPlanThreads - 1) carry = before + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    sz[0] = n_init;
    sz[1] = n_sep2;
    sz[2] = 0;
    sz[3] = n_local;
    a.len[b] = n_init + n_sep2 + n_local;
    a.ctrl[2 * b] = 1;
    a.ctrl[2 * b + 1] = total;  // slots before the compaction
  }
}

// phase 0: kept rows -> scratch at their destination; phase 1: scratch rows
// [0, len) -> cache.  grid (B * Hkv, ceil(c / rows)), 16-byte pieces.
__global__ void stream_move_kernel(StreamArgs a, int phase) {
  const int bg = blockIdx.x;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  if (!a.ctrl[2 * b]) return;
  const int per_row = a.d / 8;
  const int rows = blockDim.x / per_row;
  const int slot = blockIdx.y * rows + threadIdx.x / per_row;
  const int x = threadIdx.x % per_row;
  const int n_slots = phase == 0 ? a.ctrl[2 * b + 1] : a.len[b];
  if (slot >= n_slots) return;
  int to = slot, from = slot;
  if (phase == 0) {
    to = a.dst[(size_t)b * a.c + slot];
    if (to < 0) return;
  }
  const size_t head = ((size_t)b * a.Hkv + g) * a.c;
  const __nv_bfloat16* ks = phase == 0 ? a.K : a.Ks;
  const __nv_bfloat16* vs = phase == 0 ? a.V : a.Vs;
  __nv_bfloat16* kd = phase == 0 ? a.Ks : a.K;
  __nv_bfloat16* vd = phase == 0 ? a.Vs : a.V;
  *reinterpret_cast<uint4*>(kd + (head + to) * a.d + x * 8) =
      *reinterpret_cast<const uint4*>(ks + (head + from) * a.d + x * 8);
  *reinterpret_cast<uint4*>(vd + (head + to) * a.d + x * 8) =
      *reinterpret_cast<const uint4*>(vs + (head + from) * a.d + x * 8);
  if (g == 0 && x == 0) {
    const size_t r = (size_t)b * a.c;
    if (phase == 0) {
      a.pos_s[r + to] = a.pos[r + from];
      a.flag_s[r + to] = a.flag[r + from];
    } else {
      a.pos[r + to] = a.pos_s[r + from];
      a.flag[r + to] = a.flag_s[r + from];
    }
  }
}

}  // namespace

cudaError_t launch_stream_append(const StreamArgs& a, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  stream_append_kernel<<<a.B * a.Hkv, a.d / 8, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  stream_plan_kernel<<<a.B, kPlanThreads, 0, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int threads = 256, rows = threads / (a.d / 8);
  dim3 grid(a.B * a.Hkv, (a.c + rows - 1) / rows);
  for (int phase = 0; phase < 2; ++phase) {
    stream_move_kernel<<<grid, threads, 0, st>>>(a, phase);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace sattn
