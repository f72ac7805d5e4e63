// bwd_simt.cu -- the CUDA-core parts of the bf16 backward pass ("SepLLM",
// section 6.2: training runs the forward and the backward pass through the
// masked product).
//
//   bwd_rows_kernel        per row: D_i = dO_i . O_i and -LSE_i log2(e)
//                          (padded to whole 128-row tiles) and, since the
//                          starting-span keys j < n_start ("LM-Infinite",
//                          section 方法) are fp32 side keys in the forward and
//                          here too, P and dS of the row's sink pairs (their
//                          dq is added by the dq kernel's epilogue);
//   bwd_sink_keys_kernel   dk and dv of the sink keys: fixed-order sums over
//                          row blocks (no atomics);
//   bwd_combine_kernel     dk_j, dv_j = band-tile part + separator part (its
//                          compacted slot) + sink part, rounded to bf16.
#include <math_constants.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSinkRowBlock = 256;  // rows per partial sum of the sink-key reduction

__device__ __forceinline__ float2 tab_at(const float2* tab, int64_t pos, int half, int c) {
  return tab ? tab[pos * half + c] : make_float2(1.f, 0.f);
}
__device__ __forceinline__ void rot(float x0, float x1, float2 cs, float& y0, float& y1) {
  y0 = x0 * cs.x - x1 * cs.y;
  y1 = x1 * cs.x + x0 * cs.y;
}
__device__ __forceinline__ void rot_t(float y0, float y1, float2 cs, float& x0, float& x1) {
  x0 = y0 * cs.x + y1 * cs.y;
  x1 = y1 * cs.x - y0 * cs.y;
}
__device__ __forceinline__ float bf(const __nv_bfloat16* p, int64_t idx) { return __bfloat162float(p[idx]); }

// Per-row pass: D_i = dO_i . O_i, -LSE_i log2(e) (padded rows: 0, -inf) and,
// for the sink keys, P_ij and dS_ij.  8 lanes per row, lane l owning the
// elements c0 + e and c0 + e + D/2 for c0 = l * E, e < E = D/16.  A block is
// 32 rows of one (b, h); the group's sink V rows are staged in shared memory
// as fp32.
constexpr int kSinkStage = 16;  // sink rows staged in shared memory at a time

// 8 consecutive bf16 (16 bytes, E = 8) or 4 (8 bytes, E = 4) as floats
template <int E>
__device__ __forceinline__ void load_row_part(const __nv_bfloat16* p, float* out) {
  if constexpr (E == 8) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const float2 f = __bfloat1622float2(h[y]);
      out[2 * y] = f.x;
      out[2 * y + 1] = f.y;
    }
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int y = 0; y < 2; ++y) {
      const float2 f = __bfloat1622float2(h[y]);
      out[2 * y] = f.x;
      out[2 * y + 1] = f.y;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(256) bwd_rows_kernel(BwdArgs a) {
  constexpr int E = D / 16;  // pairs per lane
  constexpr int H = D / 2;
  __shared__ float s_sink[kSinkStage][D];  // v_j of a stage of sinks
  const int blocks_per_head = a.Tpad / 32;
  const int64_t bh = blockIdx.x / blocks_per_head;
  const int i = (int)(blockIdx.x % blocks_per_head) * 32 + (threadIdx.x >> 3);
  const int l = threadIdx.x & 7;
  const int h = (int)(bh % a.Hq), b = (int)(bh / a.Hq);
  const int g = h / (a.Hq / a.Hkv);
  const int ns_all = a.n_sink;
  const bool row_ok = i < a.T;
  const int64_t prow = bh * a.Tpad + i;
  const int c0 = l * E;
  float g0[E], g1[E];
  float dd = 0.f, nl2 = -CUDART_INF_F;
  if (row_ok) {
    const int64_t ooff = b * a.o_sb + h * a.o_sh + (int64_t)i * a.o_st;
    float o0[E], o1[E];
    load_row_part<E>(a.dO + ooff + c0, g0);
    load_row_part<E>(a.dO + ooff + c0 + H, g1);
    load_row_part<E>(a.O + ooff + c0, o0);
    load_row_part<E>(a.O + ooff + c0 + H, o1);
#pragma unroll
    for (int e = 0; e < E; ++e) dd = fmaf(g0[e], o0[e], fmaf(g1[e], o1[e], dd));
    nl2 = -a.lse[bh * a.T + i] * kLog2e;
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) g0[e] = g1[e] = 0.f;
  }
  dd += __shfl_xor_sync(0xffffffffu, dd, 1);
  dd += __shfl_xor_sync(0xffffffffu, dd, 2);
  dd += __shfl_xor_sync(0xffffffffu, dd, 4);
  if (l == 0) {
    a.Dsum[prow] = dd;
    a.nlse2[prow] = nl2;
  }
  if (ns_all == 0) return;  // uniform over the block
  const int ns = row_ok ? min(ns_all, i + 1) : 0;
  const int64_t wid = bh * a.T + i;
  for (int js = 0; js < ns_all; js += kSinkStage) {
    const int nst = min(kSinkStage, ns_all - js);
    __syncthreads();  // the previous stage is consumed
    for (int x = threadIdx.x; x < nst * D; x += blockDim.x) {
      const int jj = x / D, c = x % D, j = js + jj;
      s_sink[jj][c] = bf(a.V + b * a.v_sb + g * a.v_sh + (int64_t)j * a.v_st, c);
    }
    __syncthreads();
    // every lane of a row takes the same branches (same i, same j)
    for (int jj = 0; jj < nst && js + jj < ns; ++jj) {
      const int j = js + jj;
      float dp = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) dp = fmaf(g0[e], s_sink[jj][c0 + e], fmaf(g1[e], s_sink[jj][c0 + e + H], dp));
      dp += __shfl_xor_sync(0xffu << (threadIdx.x & 24), dp, 1);
      dp += __shfl_xor_sync(0xffu << (threadIdx.x & 24), dp, 2);
      dp += __shfl_xor_sync(0xffu << (threadIdx.x & 24), dp, 4);
      const float p = exp2f(fmaf(a.sink_z[wid * ns_all + j], a.scale_log2, nl2));
      const float ds = p * (dp - dd);
      if (l == 0) {
        a.sink_ds[wid * ns_all + j] = ds;
        a.sink_p[wid * ns_all + j] = p;
      }
    }
  }
}

// Sink-key partial sums of one row block: CTA per (b, g, row block, group of
// kSinkGroup sinks), 256 threads = 8 warps taking the block's rows of every
// query head of the group in turn; lane l owns pairs 2l, 2l + 1 (elements
// 2l, 2l+1, 2l+D/2, 2l+1+D/2; D = 128) or pair l (D = 64).  Per sink: sums
// of dS_ij R(i) q_i (uncapped), dS_ij R(L) q_i (capped), P_ij dO_i; the 8
// warps' sums are added in a fixed order through shared memory.  Writes the
// raw-frame dk part (R(j)^T of the uncapped sum plus the capped sum,
// unscaled) and the dv part of each sink.
constexpr int kSinkGroup = 4;
constexpr int kRowsInFlight = 8;  // rows per warp whose loads are issued together

// PL consecutive bf16 (one or two) as floats
template <int PL>
__device__ __forceinline__ void load_pl(const __nv_bfloat16* p, float* out) {
  if constexpr (PL == 2) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    out[0] = f.x;
    out[1] = f.y;
  } else {
    out[0] = __bfloat162float(*p);
  }
}

template <int D>
__global__ void __launch_bounds__(256) bwd_sink_keys_kernel(BwdArgs a) {
  constexpr int PL = D / 64;  // pairs per lane
  constexpr int H = D / 2;
  __shared__ float red[8][kSinkGroup][3][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_grp = (a.n_sink + kSinkGroup - 1) / kSinkGroup;
  int64_t x = blockIdx.x;
  const int sg = (int)(x % n_grp);
  x /= n_grp;
  const int rb = (int)(x % a.nRB);
  x /= a.nRB;
  const int g = (int)(x % a.Hkv), b = (int)(x / a.Hkv);
  const int rep = a.Hq / a.Hkv;
  const int j0 = sg * kSinkGroup;
  const int nj = min(kSinkGroup, a.n_sink - j0);
  float ar[kSinkGroup][2 * PL], ac[kSinkGroup][2 * PL], av[kSinkGroup][2 * PL];
#pragma unroll
  for (int q = 0; q < kSinkGroup; ++q)
#pragma unroll
    for (int e = 0; e < 2 * PL; ++e) ar[q][e] = ac[q][e] = av[q][e] = 0.f;
  const int i_lo = max(j0, rb * kSinkRowBlock), i_hi = min(a.T, (rb + 1) * kSinkRowBlock);
  float2 cl[PL];
#pragma unroll
  for (int e = 0; e < PL; ++e) cl[e] = a.L > 0 ? tab_at(a.tab, a.L, H, PL * lane + e) : make_float2(1.f, 0.f);
  // a warp takes rows i0, i0 + 8, ..., i0 + 8 (kRowsInFlight - 1) together:
  // their loads are issued before any is used
  for (int h = g * rep; h < (g + 1) * rep; ++h) {
    const int64_t bh = (int64_t)b * a.Hq + h;
    for (int i0 = i_lo + warp; i0 < i_hi; i0 += 8 * kRowsInFlight) {
      float q0[kRowsInFlight][PL], q1[kRowsInFlight][PL], d0[kRowsInFlight][PL], d1[kRowsInFlight][PL];
      float2 ti[kRowsInFlight][PL];
      float dsv[kRowsInFlight][kSinkGroup], pjv[kRowsInFlight][kSinkGroup];
#pragma unroll
      for (int u = 0; u < kRowsInFlight; ++u) {
        const int i = i0 + 8 * u;
        const int ic = i < i_hi ? i : i0;  // rows past the block: loads of row i0, results unused
        const int64_t wid = bh * a.T + ic;
        const __nv_bfloat16* qp = a.Q + b * a.q_sb + h * a.q_sh + (int64_t)ic * a.q_st + PL * lane;
        const __nv_bfloat16* gp = a.dO + b * a.o_sb + h * a.o_sh + (int64_t)ic * a.o_st + PL * lane;
        load_pl<PL>(qp, q0[u]);
        load_pl<PL>(qp + H, q1[u]);
        load_pl<PL>(gp, d0[u]);
        load_pl<PL>(gp + H, d1[u]);
#pragma unroll
        for (int e = 0; e < PL; ++e) ti[u][e] = tab_at(a.tab, ic, H, PL * lane + e);
#pragma unroll
        for (int q = 0; q < kSinkGroup; ++q) {
          const bool use = q < nj;
          dsv[u][q] = use ? a.sink_ds[wid * a.n_sink + j0 + q] : 0.f;
          pjv[u][q] = use ? a.sink_p[wid * a.n_sink + j0 + q] : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < kRowsInFlight; ++u) {
        const int i = i0 + 8 * u;
        if (i >= i_hi) break;
        float qi0[PL], qi1[PL], ql0[PL], ql1[PL];
#pragma unroll
        for (int e = 0; e < PL; ++e) {
          rot(q0[u][e], q1[u][e], ti[u][e], qi0[e], qi1[e]);
          rot(q0[u][e], q1[u][e], cl[e], ql0[e], ql1[e]);
        }
#pragma unroll
        for (int q = 0; q < kSinkGroup; ++q) {
          if (q >= nj) break;
          const int j = j0 + q;
          if (i < j) continue;
          const float ds = dsv[u][q];
          const float pj = pjv[u][q];
          const bool capped = a.L > 0 && (i - j) > a.L;
#pragma unroll
          for (int e = 0; e < PL; ++e) {
            if (capped) {
              ac[q][e] = fmaf(ds, ql0[e], ac[q][e]);
              ac[q][PL + e] = fmaf(ds, ql1[e], ac[q][PL + e]);
            } else {
              ar[q][e] = fmaf(ds, qi0[e], ar[q][e]);
              ar[q][PL + e] = fmaf(ds, qi1[e], ar[q][PL + e]);
            }
            av[q][e] = fmaf(pj, d0[u][e], av[q][e]);
            av[q][PL + e] = fmaf(pj, d1[u][e], av[q][PL + e]);
          }
        }
      }
    }
  }
  // fixed-order reduction over the 8 warps
#pragma unroll
  for (int q = 0; q < kSinkGroup; ++q)
#pragma unroll
    for (int e = 0; e < PL; ++e) {
      const int c = PL * lane + e;
      red[warp][q][0][c] = ar[q][e];
      red[warp][q][0][c + H] = ar[q][PL + e];
      red[warp][q][1][c] = ac[q][e];
      red[warp][q][1][c + H] = ac[q][PL + e];
      red[warp][q][2][c] = av[q][e];
      red[warp][q][2][c + H] = av[q][PL + e];
    }
  __syncthreads();
  for (int t = threadIdx.x; t < nj * H; t += blockDim.x) {
    const int q = t / H, p = t % H, j = j0 + q;
    float r0 = 0.f, r1 = 0.f, c0 = 0.f, c1 = 0.f, v0 = 0.f, v1 = 0.f;
    for (int w = 0; w < 8; ++w) {
      r0 += red[w][q][0][p];
      r1 += red[w][q][0][p + H];
      c0 += red[w][q][1][p];
      c1 += red[w][q][1][p + H];
      v0 += red[w][q][2][p];
      v1 += red[w][q][2][p + H];
    }
    float x0, x1;
    rot_t(r0, r1, tab_at(a.tab, j, H, p), x0, x1);
    float* part = a.sink_part + ((((int64_t)b * a.Hkv + g) * a.n_sink + j) * a.nRB + rb) * 2 * D;
    part[p] = x0 + c0;
    part[p + H] = x1 + c1;
    part[D + p] = v0;
    part[D + p + H] = v1;
  }
}

// one thread per 8 consecutive elements of one key row
__global__ void bwd_combine_kernel(BwdArgs a) {
  const int per_row = a.d / 8;
  const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)a.B * a.Hkv * a.T * per_row;
  if (tid >= total) return;
  const int c0 = (int)(tid % per_row) * 8;
  const int64_t key = tid / per_row;
  const int j = (int)(key % a.T);
  const int64_t bg = key / a.T;
  const int g = (int)(bg % a.Hkv), b = (int)(bg / a.Hkv);
  float k[8], v[8];
  const float* kb = a.dk_band + key * a.d + c0;
  const float* vb = a.dv_band + key * a.d + c0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    k[e] = kb[e];
    v[e] = vb[e];
  }
  if (a.gather && j >= a.n_start) {
    const uint2 wd = a.sep_words[(size_t)b * (a.T / 32 + 1) + (j >> 5)];
    if ((wd.y >> (j & 31)) & 1u) {  // j is a separator: its compacted slot r
      const int r = (int)wd.x + __popc(wd.y & ((1u << (j & 31)) - 1u));
      const float* ks = a.dk_sep + (bg * a.Tpad + r) * a.d + c0;
      const float* vs = a.dv_sep + (bg * a.Tpad + r) * a.d + c0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        k[e] += ks[e];
        v[e] += vs[e];
      }
    }
  }
  if (j < a.n_sink) {
    const float scale = rsqrtf((float)a.d);
    const float* part = a.sink_part + (size_t)((bg * a.n_sink + j) * a.nRB) * 2 * a.d;
    for (int rb = 0; rb < a.nRB; ++rb) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        k[e] = fmaf(part[(size_t)rb * 2 * a.d + c0 + e], scale, k[e]);
        v[e] += part[(size_t)rb * 2 * a.d + a.d + c0 + e];
      }
    }
  }
  __nv_bfloat16* dk = a.dK + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st + c0;
  __nv_bfloat16* dv = a.dV + b * a.v_sb + g * a.v_sh + (int64_t)j * a.v_st + c0;
  uint4 ko, vo;
  ko.x = pack_bf16x2(k[0], k[1]);
  ko.y = pack_bf16x2(k[2], k[3]);
  ko.z = pack_bf16x2(k[4], k[5]);
  ko.w = pack_bf16x2(k[6], k[7]);
  vo.x = pack_bf16x2(v[0], v[1]);
  vo.y = pack_bf16x2(v[2], v[3]);
  vo.z = pack_bf16x2(v[4], v[5]);
  vo.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(dk) = ko;
  *reinterpret_cast<uint4*>(dv) = vo;
}

}  // namespace

int bwd_sink_row_block() { return kSinkRowBlock; }

cudaError_t launch_bwd_rows(const BwdArgs& a, cudaStream_t st) {
  const int64_t blocks = (int64_t)a.B * a.Hq * (a.Tpad / 32);
  if (blocks == 0) return cudaSuccess;
  if (a.d == 128) {
    bwd_rows_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(a);
  } else if (a.d == 64) {
    bwd_rows_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_sink_keys(const BwdArgs& a, cudaStream_t st) {
  const int n_grp = (a.n_sink + kSinkGroup - 1) / kSinkGroup;
  const int64_t blocks = (int64_t)a.B * a.Hkv * a.nRB * n_grp;
  if (blocks == 0 || a.n_sink == 0) return cudaSuccess;
  if (a.d == 128)
    bwd_sink_keys_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(a);
  else if (a.d == 64)
    bwd_sink_keys_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_bwd_combine(const BwdArgs& a, cudaStream_t st) {
  const int64_t total = (int64_t)a.B * a.Hkv * a.T * (a.d / 8);
  if (total == 0) return cudaSuccess;
  bwd_combine_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace sattn
