// prep.cu -- K1: rotary table and the elementwise prep pass.
//
// Rotary convention: rotate-half; pair (c, c + d/2) turns by the angle
// p * theta^(-2c/d).  The capped logit ("LM-Infinite", section 方法, RoPE
// realisation of d'_ij = min(d_ij, L)) needs, besides R(i) q_i and R(j) k_j,
// the query rotated to the cap, R(L) q_i, paired with the unrotated key.
//
// Outputs (all optional): Qr = R(i) q_i, Qc = R(L) q_i, Kr = R(j) k_j as bf16
// tensor-core operands; the fp32 logits of the starting-span ("sink") keys,
// computed from fp32 rotations of the exact inputs so that the large sink
// logits do not inherit bf16 operand rounding; and per (batch, kv head) the
// largest key norm, used by the top-k selector to bound bf16 scoring error.
//
// Layout of the work: one block = 32 consecutive rows of one head (8 warps,
// 4 rows each); lane l owns the pairs c = l*PP .. l*PP+PP-1 (PP = d/64), so a
// row's loads and stores are 128-byte coalesced per half.  Sink keys are
// staged once per block in shared memory (raw and rotated, fp32).
#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"

namespace sattn {

namespace {

constexpr int kRowsPerBlock = 32;
constexpr int kPrepThreads = 256;
constexpr int kMaxSmemSinks = 16;

__global__ void rope_table_kernel(float2* tab, int npos, int half, int d, double theta) {
  __shared__ double inv_freq[128];
  for (int c = threadIdx.x; c < half; c += blockDim.x) inv_freq[c] = pow(theta, -2.0 * (double)c / (double)d);
  __syncthreads();
  const int64_t n = (int64_t)npos * half;
  for (int64_t x = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; x < n; x += (int64_t)gridDim.x * blockDim.x) {
    const int p = (int)(x / half);
    const int c = (int)(x % half);
    double s, co;
    sincos((double)p * inv_freq[c], &s, &co);
    tab[x] = make_float2((float)co, (float)s);
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// PP consecutive bf16 of a row starting at element c -> floats
template <int PP>
__device__ __forceinline__ void load_pp(const __nv_bfloat16* p, float* out) {
  if constexpr (PP == 2) {
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    out[0] = v.x;
    out[1] = v.y;
  } else {
    out[0] = __bfloat162float(*p);
  }
}

template <int PP>
__device__ __forceinline__ void store_pp(__nv_bfloat16* p, const float* v) {
  if constexpr (PP == 2) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v[0], v[1]);
  } else {
    *p = __float2bfloat16_rn(v[0]);
  }
}

template <int PP>
__device__ __forceinline__ void load_tab(const float2* tab, int64_t pos, int half, int c, float* cs, float* sn) {
  if (!tab) {
#pragma unroll
    for (int e = 0; e < PP; ++e) {
      cs[e] = 1.f;
      sn[e] = 0.f;
    }
    return;
  }
  const float2* t = tab + pos * half + c;
  if constexpr (PP == 2) {
    const float4 v = *reinterpret_cast<const float4*>(t);
    cs[0] = v.x;
    sn[0] = v.y;
    cs[1] = v.z;
    sn[1] = v.w;
  } else {
    const float2 v = *t;
    cs[0] = v.x;
    sn[0] = v.y;
  }
}

// grid (ceil(T/32), H, B) for the query part (blockIdx.z < B) followed by
// the key part (blockIdx.z >= B, head = blockIdx.y < Hkv)
template <int PP>
__global__ void __launch_bounds__(kPrepThreads) prep_kernel(PrepArgs a) {
  __shared__ float s_sink_raw[kMaxSmemSinks][128];
  __shared__ float s_sink_rot[kMaxSmemSinks][128];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = a.d / 2;
  const int c0 = lane * PP;
  const bool key_part = blockIdx.z >= (unsigned)a.B;
  const int b = key_part ? blockIdx.z - a.B : blockIdx.z;
  const int h = blockIdx.y;
  const int row0 = blockIdx.x * kRowsPerBlock;
  const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.Q);
  const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(a.K);

  if (key_part) {
    if (h >= a.Hkv) return;
    constexpr int kRowsPerWarp = kRowsPerBlock / (kPrepThreads / 32);
    float k0[kRowsPerWarp][PP], k1[kRowsPerWarp][PP], cs[kRowsPerWarp][PP], sn[kRowsPerWarp][PP];
#pragma unroll
    for (int x = 0; x < kRowsPerWarp; ++x) {
      const int j = min(row0 + warp + x * (kPrepThreads / 32), a.T - 1);
      const __nv_bfloat16* kp = K + b * a.k_sb + h * a.k_sh + (int64_t)j * a.k_st;
      load_pp<PP>(kp + c0, k0[x]);
      load_pp<PP>(kp + c0 + half, k1[x]);
      load_tab<PP>(a.tab, j, half, c0, cs[x], sn[x]);
    }
#pragma unroll
    for (int x = 0; x < kRowsPerWarp; ++x) {
      const int j = row0 + warp + x * (kPrepThreads / 32);
      if (j >= a.T) break;
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < PP; ++e) ss = fmaf(k0[x][e], k0[x][e], fmaf(k1[x][e], k1[x][e], ss));
      if (a.Kr) {
        float r0[PP], r1[PP];
#pragma unroll
        for (int e = 0; e < PP; ++e) {
          r0[e] = k0[x][e] * cs[x][e] - k1[x][e] * sn[x][e];
          r1[e] = k1[x][e] * cs[x][e] + k0[x][e] * sn[x][e];
        }
        __nv_bfloat16* kr = a.Kr + (((int64_t)b * a.Hkv + h) * a.T + j) * a.d;
        store_pp<PP>(kr + c0, r0);
        store_pp<PP>(kr + c0 + half, r1);
      }
      if (a.kmax) {
        ss = warp_sum(ss);
        if (lane == 0) atomicMax(a.kmax + (size_t)b * a.Hkv + h, __float_as_uint(sqrtf(ss)));
      }
    }
    return;
  }

  // ---- query part ----
  const int g = h / (a.Hq / a.Hkv);
  const int n_sink = a.sink_z ? a.n_sink : 0;
  const bool sinks_in_smem = n_sink > 0 && n_sink <= kMaxSmemSinks;
  if (sinks_in_smem) {
    // raw and rotated sink keys of this (b, kv head), fp32
    for (int x = threadIdx.x; x < n_sink * half; x += kPrepThreads) {
      const int j = x / half, c = x % half;
      const __nv_bfloat16* kp = K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st;
      const float k0 = __bfloat162float(kp[c]), k1 = __bfloat162float(kp[c + half]);
      const float2 t = a.tab ? a.tab[(int64_t)j * half + c] : make_float2(1.f, 0.f);
      s_sink_raw[j][c] = k0;
      s_sink_raw[j][c + half] = k1;
      s_sink_rot[j][c] = k0 * t.x - k1 * t.y;
      s_sink_rot[j][c + half] = k1 * t.x + k0 * t.y;
    }
    __syncthreads();
  }
  const bool need_qc = a.Qc != nullptr || n_sink > 0;
  float lc[PP], ls[PP];
  if (need_qc) load_tab<PP>(a.L > 0 ? a.tab : nullptr, a.L, half, c0, lc, ls);
  constexpr int kRowsPerWarp = kRowsPerBlock / (kPrepThreads / 32);
  float xa[kRowsPerWarp][PP], xb[kRowsPerWarp][PP], ca[kRowsPerWarp][PP], sa[kRowsPerWarp][PP];
#pragma unroll
  for (int x = 0; x < kRowsPerWarp; ++x) {
    const int i = min(row0 + warp + x * (kPrepThreads / 32), a.T - 1);
    const __nv_bfloat16* qp = Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st;
    load_pp<PP>(qp + c0, xa[x]);
    load_pp<PP>(qp + c0 + half, xb[x]);
    load_tab<PP>(a.tab, i, half, c0, ca[x], sa[x]);
  }
#pragma unroll
  for (int x = 0; x < kRowsPerWarp; ++x) {
    const int i = row0 + warp + x * (kPrepThreads / 32);
    if (i >= a.T) break;
    float r0[PP], r1[PP], q0[PP], q1[PP];
#pragma unroll
    for (int e = 0; e < PP; ++e) {
      r0[e] = xa[x][e] * ca[x][e] - xb[x][e] * sa[x][e];
      r1[e] = xb[x][e] * ca[x][e] + xa[x][e] * sa[x][e];
      q0[e] = xa[x][e] * lc[e] - xb[x][e] * ls[e];
      q1[e] = xb[x][e] * lc[e] + xa[x][e] * ls[e];
    }
    const int64_t orow = (((int64_t)b * a.Hq + h) * a.T + i) * a.d;
    if (a.Qr) {
      store_pp<PP>(a.Qr + orow + c0, r0);
      store_pp<PP>(a.Qr + orow + c0 + half, r1);
    }
    if (a.Qc) {
      store_pp<PP>(a.Qc + orow + c0, q0);
      store_pp<PP>(a.Qc + orow + c0 + half, q1);
    }
    if (n_sink > 0) {
      const int64_t zrow = (((int64_t)b * a.Hq + h) * a.T + i) * n_sink;
      for (int j0 = 0; j0 < n_sink; j0 += 32) {
        float mine = -CUDART_INF_F;
        const int jn = min(32, n_sink - j0);
        for (int jj = 0; jj < jn; ++jj) {
          const int j = j0 + jj;
          float z = -CUDART_INF_F;
          if (j <= i) {
            const bool capped = a.L > 0 && (i - j) > a.L;
            float acc = 0.f;
            if (sinks_in_smem) {
              const float* kv = capped ? s_sink_raw[j] : s_sink_rot[j];
#pragma unroll
              for (int e = 0; e < PP; ++e) {
                acc = fmaf(capped ? q0[e] : r0[e], kv[c0 + e], acc);
                acc = fmaf(capped ? q1[e] : r1[e], kv[c0 + e + half], acc);
              }
            } else {
              const __nv_bfloat16* kp = K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st;
              float k0[PP], k1[PP], kc[PP], ks[PP];
              load_pp<PP>(kp + c0, k0);
              load_pp<PP>(kp + c0 + half, k1);
              load_tab<PP>(a.tab, j, half, c0, kc, ks);
#pragma unroll
              for (int e = 0; e < PP; ++e) {
                if (capped) {
                  acc = fmaf(q0[e], k0[e], fmaf(q1[e], k1[e], acc));
                } else {
                  acc = fmaf(r0[e], k0[e] * kc[e] - k1[e] * ks[e], acc);
                  acc = fmaf(r1[e], k1[e] * kc[e] + k0[e] * ks[e], acc);
                }
              }
            }
            z = warp_sum(acc);
          }
          if (lane == jj) mine = z;
        }
        if (lane < jn) a.sink_z[zrow + j0 + lane] = mine;
      }
    }
  }
}

}  // namespace

cudaError_t launch_rope_table(float2* tab, int npos, int d, double theta, cudaStream_t st) {
  const int half = d / 2;
  const int64_t n = (int64_t)npos * half;
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>((n + threads - 1) / threads, 148 * 16);
  rope_table_kernel<<<(unsigned)blocks, threads, 0, st>>>(tab, npos, half, d, theta);
  return cudaGetLastError();
}

cudaError_t launch_prep(const PrepArgs& a, cudaStream_t st) {
  if (a.f32) return cudaErrorInvalidValue;  // the fp32 path rotates inside its own kernel
  if (a.B == 0 || a.T == 0) return cudaSuccess;
  dim3 grid((a.T + kRowsPerBlock - 1) / kRowsPerBlock, std::max(a.Hq, a.Hkv), 2 * a.B);
  if (a.d == 128)
    prep_kernel<2><<<grid, kPrepThreads, 0, st>>>(a);
  else if (a.d == 64)
    prep_kernel<1><<<grid, kPrepThreads, 0, st>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace sattn
