// bwd_topk.cu -- the top-k keys' part of the bf16 backward pass.
//
// The optional top-k middle tokens ("LM-Infinite", section 方法, optional
// top-k paragraph) are fp32 side keys in the forward, so their gradients are
// formed here on the CUDA cores, with the selection a constant of the
// backward pass (as for the oracle).  For a selected pair (i, j) with
// P_ij = exp(s_ij - LSE_i), dS_ij = P_ij (dO_i . v_j - D_i) and dz = dS / sqrt(d):
//   capped pair (L > 0, i - j > L; z = <R(L) q_i, k_j>):
//     dq_i += R(L)^T dz k_j,      dk_j += dz R(L) q_i;
//   uncapped pair (z = <R(i) q_i, R(j) k_j>):
//     dq_i += R(i)^T dz R(j) k_j, dk_j += R(j)^T dz R(i) q_i;
//   dv_j += P_ij dO_i.
//
//   bwd_topk_rows_kernel   a warp per query row: the row's k pairs, their P
//                          and dS (kept for the key side) and the row's dq
//                          part, added into the fp32 side dq that the dq
//                          kernel's epilogue adds;
//   bwd_topk_count_kernel  selections per key (integer atomics: the counts
//                          are exact whatever the order);
//   bwd_topk_scan_kernel   a block per (batch, kv head): exclusive prefix sum
//                          of the counts, each key's offset in the segment;
//   bwd_topk_fill_kernel   each selection's code (head, row, slot) into its
//                          key's slots (the order within a key is arbitrary);
//   bwd_topk_keys_kernel   a warp per selected key: orders the key's codes by
//                          rank (ascending head, row, slot), then sums dk and
//                          dv in that order and adds them to the key's
//                          band-tile parts.
// No floating-point atomics: the result is the same bit for bit on repeat.
#include <math_constants.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

constexpr int kScanThreads = 1024;

__device__ __forceinline__ float warp_sum32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float2 tab_at(const float2* tab, int64_t pos, int half, int c) {
  return tab ? tab[pos * half + c] : make_float2(1.f, 0.f);
}

// A lane owns the rotary pairs c = lane * PL + e (e < PL) of a row: elements
// c and c + D/2.
template <int D>
struct RowPart {
  static constexpr int PL = D / 64;
  static constexpr int H = D / 2;
  float x0[PL], x1[PL];
  __device__ __forceinline__ void load(const __nv_bfloat16* row, int lane) {
#pragma unroll
    for (int e = 0; e < PL; ++e) {
      x0[e] = __bfloat162float(row[lane * PL + e]);
      x1[e] = __bfloat162float(row[lane * PL + e + H]);
    }
  }
  // R(pos) x
  __device__ __forceinline__ RowPart rotated(const float2* tab, int64_t pos, int lane) const {
    RowPart r;
#pragma unroll
    for (int e = 0; e < PL; ++e) {
      const float2 cs = tab_at(tab, pos, H, lane * PL + e);
      r.x0[e] = x0[e] * cs.x - x1[e] * cs.y;
      r.x1[e] = x1[e] * cs.x + x0[e] * cs.y;
    }
    return r;
  }
  // R(pos)^T x
  __device__ __forceinline__ RowPart rotated_back(const float2* tab, int64_t pos, int lane) const {
    RowPart r;
#pragma unroll
    for (int e = 0; e < PL; ++e) {
      const float2 cs = tab_at(tab, pos, H, lane * PL + e);
      r.x0[e] = x0[e] * cs.x + x1[e] * cs.y;
      r.x1[e] = x1[e] * cs.x - x0[e] * cs.y;
    }
    return r;
  }
  __device__ __forceinline__ float dot(const RowPart& o) const {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < PL; ++e) s = fmaf(x0[e], o.x0[e], fmaf(x1[e], o.x1[e], s));
    return s;
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int e = 0; e < PL; ++e) x0[e] = x1[e] = 0.f;
  }
  __device__ __forceinline__ void axpy(float a, const RowPart& o) {
#pragma unroll
    for (int e = 0; e < PL; ++e) {
      x0[e] = fmaf(a, o.x0[e], x0[e]);
      x1[e] = fmaf(a, o.x1[e], x1[e]);
    }
  }
};

template <int D>
__global__ void __launch_bounds__(256) bwd_topk_rows_kernel(BwdArgs a, int add_side) {
  using RP = RowPart<D>;
  const int lane = threadIdx.x & 31;
  const int64_t nrows = (int64_t)a.B * a.Hq * a.T;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= nrows) return;  // whole warps only: no block-wide barrier follows
  const int i = (int)(row % a.T);
  const int64_t bh = row / a.T;
  const int h = (int)(bh % a.Hq), b = (int)(bh / a.Hq);
  const int g = h / (a.Hq / a.Hkv);
  const int k = a.topk;
  const float scale = rsqrtf((float)a.d);
  const float dd = a.Dsum[bh * a.Tpad + i];
  const float nl2 = a.nlse2[bh * a.Tpad + i];
  RP q, go;
  q.load(a.Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st, lane);
  go.load(a.dO + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st, lane);
  const RP qi = q.rotated(a.tab, i, lane);
  const RP qc = q.rotated(a.tab, a.L > 0 ? a.L : 0, lane);
  const float slope = a.alibi ? alibi_slope_qk(h, a.Hq, a.d) : 0.f;
  RP acc_r, acc_c;  // dS-weighted keys of the uncapped (rotated by R(j)) and capped pairs
  acc_r.zero();
  acc_c.zero();
  for (int x = 0; x < k; ++x) {
    const int j = a.tk_idx[row * k + x];
    float ds = 0.f, p = 0.f;
    if (j >= 0 && j <= i) {  // uniform over the warp
      const bool capped = a.L > 0 && (i - j) > a.L;
      RP kr, vr;
      kr.load(a.K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st, lane);
      vr.load(a.V + b * a.v_sb + g * a.v_sh + (int64_t)j * a.v_st, lane);
      const RP ks = capped ? kr : kr.rotated(a.tab, j, lane);
      const float z = warp_sum32(capped ? qc.dot(ks) : qi.dot(ks));
      const int dist = a.L > 0 ? min(i - j, a.L) : (i - j);
      const float s2 = (z - slope * (float)dist) * a.scale_log2;  // log2 units
      p = exp2f(s2 + nl2);
      const float dp = warp_sum32(go.dot(vr));
      ds = p * (dp - dd);
      if (capped) acc_c.axpy(ds, ks);
      else acc_r.axpy(ds, ks);
    }
    if (lane == 0) {
      a.tk_ds[row * k + x] = ds;
      a.tk_p[row * k + x] = p;
    }
  }
  // back to the raw frame: R(i)^T of the uncapped sum, R(L)^T of the capped one
  const RP br = acc_r.rotated_back(a.tab, i, lane);
  const RP bc = acc_c.rotated_back(a.tab, a.L > 0 ? a.L : 0, lane);
  float* side = a.dq_side + row * a.d;
#pragma unroll
  for (int e = 0; e < RP::PL; ++e) {
    const int c = lane * RP::PL + e;
    const float v0 = (br.x0[e] + bc.x0[e]) * scale, v1 = (br.x1[e] + bc.x1[e]) * scale;
    side[c] = add_side ? side[c] + v0 : v0;
    side[c + RP::H] = add_side ? side[c + RP::H] + v1 : v1;
  }
}

// one thread per (row, slot)
__global__ void bwd_topk_count_kernel(BwdArgs a) {
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t n = (int64_t)a.B * a.Hq * a.T * a.topk;
  if (t >= n) return;
  const int64_t row = t / a.topk;
  const int i = (int)(row % a.T);
  const int64_t bh = row / a.T;
  const int h = (int)(bh % a.Hq), b = (int)(bh / a.Hq);
  const int j = a.tk_idx[t];
  if (j < 0 || j > i) return;
  const int g = h / (a.Hq / a.Hkv);
  atomicAdd(a.tk_cnt + ((int64_t)b * a.Hkv + g) * a.T + j, 1);
}

// a block per (batch, kv head): exclusive prefix sum of the counts of the T
// keys; the offsets go to tk_off and, as fill cursors, to tk_cur
__global__ void __launch_bounds__(kScanThreads) bwd_topk_scan_kernel(BwdArgs a) {
  __shared__ int warp_tot[kScanThreads / 32];
  __shared__ int carry;
  const int64_t seg = blockIdx.x;
  const int* cnt = a.tk_cnt + seg * a.T;
  int* off = a.tk_off + seg * a.T;
  int* cur = a.tk_cur + seg * a.T;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < a.T; base += kScanThreads) {
    const int j = base + threadIdx.x;
    const int c = j < a.T ? cnt[j] : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int v = warp_tot[lane];
      int sc = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, sc, o);
        if (lane >= o) sc += y;
      }
      warp_tot[lane] = sc - v;
    }
    __syncthreads();
    const int ex = carry + warp_tot[warp] + incl - c;
    if (j < a.T) {
      off[j] = ex;
      cur[j] = ex;
    }
    __syncthreads();  // carry and warp_tot are consumed
    if (threadIdx.x == kScanThreads - 1) carry = ex + c;
    __syncthreads();
  }
}

// one thread per (row, slot): the selection's code (local head, row, slot)
// into a slot of its key
__global__ void bwd_topk_fill_kernel(BwdArgs a) {
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t n = (int64_t)a.B * a.Hq * a.T * a.topk;
  if (t >= n) return;
  const int x = (int)(t % a.topk);
  const int64_t row = t / a.topk;
  const int i = (int)(row % a.T);
  const int64_t bh = row / a.T;
  const int h = (int)(bh % a.Hq), b = (int)(bh / a.Hq);
  const int j = a.tk_idx[t];
  if (j < 0 || j > i) return;
  const int rep = a.Hq / a.Hkv;
  const int g = h / rep;
  const int64_t seg = (int64_t)b * a.Hkv + g;
  const int pos = atomicAdd(a.tk_cur + seg * a.T + j, 1);
  a.tk_code[seg * (int64_t)rep * a.T * a.topk + pos] = ((h - g * rep) * a.T + i) * a.topk + x;
}

// a warp per key (batch, kv head, j) selected at least once
template <int D>
__global__ void __launch_bounds__(256) bwd_topk_keys_kernel(BwdArgs a) {
  using RP = RowPart<D>;
  const int lane = threadIdx.x & 31;
  const int64_t nkeys = (int64_t)a.B * a.Hkv * a.T;
  const int64_t key = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (key >= nkeys) return;
  const int c = a.tk_cnt[key];
  if (c == 0) return;  // uniform over the warp
  const int j = (int)(key % a.T);
  const int64_t seg = key / a.T;
  const int g = (int)(seg % a.Hkv), b = (int)(seg / a.Hkv);
  const int rep = a.Hq / a.Hkv;
  const int k = a.topk;
  const int64_t base = seg * (int64_t)rep * a.T * k + a.tk_off[key];
  const int* code = a.tk_code + base;
  int* sorted = a.tk_sorted + base;
  // order the key's codes: an entry's place is the number of smaller codes
  for (int e = lane; e < c; e += 32) {
    const int ce = code[e];
    int rank = 0;
    for (int f = 0; f < c; ++f) rank += code[f] < ce ? 1 : 0;
    sorted[rank] = ce;
  }
  __syncwarp();
  const float scale = rsqrtf((float)a.d);
  RP acc_r, acc_c, acc_v;
  acc_r.zero();
  acc_c.zero();
  acc_v.zero();
  for (int e = 0; e < c; ++e) {
    const int ce = sorted[e];
    const int x = ce % k;
    const int hl = ce / k / a.T;
    const int i = (ce / k) % a.T;
    const int h = g * rep + hl;
    const int64_t row = ((int64_t)b * a.Hq + h) * a.T + i;
    const float ds = a.tk_ds[row * k + x];
    const float p = a.tk_p[row * k + x];
    const bool capped = a.L > 0 && (i - j) > a.L;
    RP q, go;
    q.load(a.Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st, lane);
    go.load(a.dO + b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st, lane);
    if (capped) acc_c.axpy(ds, q.rotated(a.tab, a.L, lane));
    else acc_r.axpy(ds, q.rotated(a.tab, i, lane));
    acc_v.axpy(p, go);
  }
  const RP br = acc_r.rotated_back(a.tab, j, lane);
  float* dk = a.dk_band + key * a.d;
  float* dv = a.dv_band + key * a.d;
#pragma unroll
  for (int e = 0; e < RP::PL; ++e) {
    const int cc = lane * RP::PL + e;
    dk[cc] += (br.x0[e] + acc_c.x0[e]) * scale;
    dk[cc + RP::H] += (br.x1[e] + acc_c.x1[e]) * scale;
    dv[cc] += acc_v.x0[e];
    dv[cc + RP::H] += acc_v.x1[e];
  }
}

}  // namespace

cudaError_t launch_bwd_topk_rows(const BwdArgs& a, bool add_side, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.Hq * a.T;
  if (rows == 0 || a.topk == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  if (a.d == 128) bwd_topk_rows_kernel<128><<<blocks, 256, 0, st>>>(a, add_side ? 1 : 0);
  else if (a.d == 64) bwd_topk_rows_kernel<64><<<blocks, 256, 0, st>>>(a, add_side ? 1 : 0);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_bwd_topk_keys(const BwdArgs& a, cudaStream_t st) {
  const int64_t sel = (int64_t)a.B * a.Hq * a.T * a.topk;
  const int64_t keys = (int64_t)a.B * a.Hkv * a.T;
  if (sel == 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(a.tk_cnt, 0, keys * sizeof(int), st);
  if (e != cudaSuccess) return e;
  bwd_topk_count_kernel<<<(unsigned)((sel + 255) / 256), 256, 0, st>>>(a);
  bwd_topk_scan_kernel<<<(unsigned)((int64_t)a.B * a.Hkv), kScanThreads, 0, st>>>(a);
  bwd_topk_fill_kernel<<<(unsigned)((sel + 255) / 256), 256, 0, st>>>(a);
  const unsigned blocks = (unsigned)((keys + 7) / 8);
  if (a.d == 128) bwd_topk_keys_kernel<128><<<blocks, 256, 0, st>>>(a);
  else if (a.d == 64) bwd_topk_keys_kernel<64><<<blocks, 256, 0, st>>>(a);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace sattn
