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
// Work layout (HBM-bound): a thread owns 8 consecutive rotary pairs of one
// row -- one 16-byte load from each half of the row, four 16-byte table
// loads, two 16-byte stores -- so d/16 threads cover a row (8 for d = 128)
// and a 256-thread block covers 256/(d/16) rows per step.  A block walks
// kRowsPerBlock rows of one head; the sink keys of that head are staged
// once per block in shared memory (raw and rotated, fp32).
#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"

namespace sattn {

namespace {

constexpr int kPrepThreads = 256;
constexpr int kRowsPerBlock = 256;
constexpr int kMaxSmemSinks = 16;
constexpr int kPairsPerThread = 8;

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

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 v = __bfloat1622float2(h[e]);
    f[2 * e] = v.x;
    f[2 * e + 1] = v.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
  return u;
}

// cos/sin of 8 consecutive pairs c0..c0+7 at position pos (identity without a table)
__device__ __forceinline__ void load_tab8(const float2* tab, int64_t pos, int half, int c0, float* cs, float* sn) {
  if (!tab) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      cs[e] = 1.f;
      sn[e] = 0.f;
    }
    return;
  }
  const float4* t = reinterpret_cast<const float4*>(tab + pos * half + c0);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float4 v = t[e];
    cs[2 * e] = v.x;
    sn[2 * e] = v.y;
    cs[2 * e + 1] = v.z;
    sn[2 * e + 1] = v.w;
  }
}

// grid (ceil(T / kRowsPerBlock), H, 2B): blockIdx.z < B -> query rows of head
// blockIdx.y; blockIdx.z >= B -> key rows of kv head blockIdx.y (< Hkv)
__global__ void __launch_bounds__(kPrepThreads, 4) prep_kernel(PrepArgs a) {
  __shared__ float s_sink_raw[kMaxSmemSinks][128];
  __shared__ float s_sink_rot[kMaxSmemSinks][128];
  __shared__ float s_lc[64], s_ls[64];  // cos/sin of the rotation to the cap L
  const int half = a.d / 2;
  const int tpr = half / kPairsPerThread;  // threads per row: 8 (d=128) or 4 (d=64)
  const int rows_per_step = kPrepThreads / tpr;
  const int sub = threadIdx.x % tpr;       // which 8-pair chunk of the row
  const int c0 = sub * kPairsPerThread;
  const bool key_part = blockIdx.z >= (unsigned)a.B;
  const int b = key_part ? blockIdx.z - a.B : blockIdx.z;
  const int h = blockIdx.y;
  const int row0 = blockIdx.x * kRowsPerBlock;
  const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.Q);
  const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(a.K);
  // lanes of this thread's row group (8 or 4 consecutive lanes)
  const unsigned grp_mask = (tpr == 8) ? (0xffu << (threadIdx.x & 24)) : (0xfu << (threadIdx.x & 28));

  if (key_part) {
    if (h >= a.Hkv) return;
    for (int rr = threadIdx.x / tpr; rr < kRowsPerBlock; rr += rows_per_step) {
      const int j = row0 + rr;
      if (j >= a.T) break;
      const __nv_bfloat16* kp = K + b * a.k_sb + h * a.k_sh + (int64_t)j * a.k_st;
      float k0[8], k1[8], cs[8], sn[8];
      unpack8(*reinterpret_cast<const uint4*>(kp + c0), k0);
      unpack8(*reinterpret_cast<const uint4*>(kp + c0 + half), k1);
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(k0[e], k0[e], fmaf(k1[e], k1[e], ss));
      if (a.Kr) {
        load_tab8(a.tab, j, half, c0, cs, sn);
        float r0[8], r1[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          r0[e] = k0[e] * cs[e] - k1[e] * sn[e];
          r1[e] = k1[e] * cs[e] + k0[e] * sn[e];
        }
        __nv_bfloat16* kr = a.Kr + (((int64_t)b * a.Hkv + h) * a.T + j) * a.d;
        *reinterpret_cast<uint4*>(kr + c0) = pack8(r0);
        *reinterpret_cast<uint4*>(kr + c0 + half) = pack8(r1);
      }
      if (a.kmax) {
        for (int o = tpr / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(grp_mask, ss, o);
        if (sub == 0) atomicMax(a.kmax + (size_t)b * a.Hkv + h, __float_as_uint(sqrtf(ss)));
      }
    }
    return;
  }

  // ---- query rows ----
  const int g = h / (a.Hq / a.Hkv);
  const int n_sink = a.sink_z ? a.n_sink : 0;
  const bool sinks_in_smem = n_sink > 0 && n_sink <= kMaxSmemSinks;
  for (int c = threadIdx.x; c < half; c += kPrepThreads) {
    const float2 t = (a.L > 0 && a.tab) ? a.tab[(int64_t)a.L * half + c] : make_float2(1.f, 0.f);
    s_lc[c] = t.x;
    s_ls[c] = t.y;
  }
  if (sinks_in_smem) {
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
  }
  __syncthreads();
  for (int rr = threadIdx.x / tpr; rr < kRowsPerBlock; rr += rows_per_step) {
    const int i = row0 + rr;
    if (i >= a.T) break;
    const __nv_bfloat16* qp = Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st;
    float x0[8], x1[8], cs[8], sn[8], r0[8], r1[8], q0[8], q1[8];
    unpack8(*reinterpret_cast<const uint4*>(qp + c0), x0);
    unpack8(*reinterpret_cast<const uint4*>(qp + c0 + half), x1);
    load_tab8(a.tab, i, half, c0, cs, sn);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      r0[e] = x0[e] * cs[e] - x1[e] * sn[e];
      r1[e] = x1[e] * cs[e] + x0[e] * sn[e];
      q0[e] = x0[e] * s_lc[c0 + e] - x1[e] * s_ls[c0 + e];
      q1[e] = x1[e] * s_lc[c0 + e] + x0[e] * s_ls[c0 + e];
    }
    const int64_t orow = (((int64_t)b * a.Hq + h) * a.T + i) * a.d;
    if (a.Qr) {
      *reinterpret_cast<uint4*>(a.Qr + orow + c0) = pack8(r0);
      *reinterpret_cast<uint4*>(a.Qr + orow + c0 + half) = pack8(r1);
    }
    if (a.Qc) {
      *reinterpret_cast<uint4*>(a.Qc + orow + c0) = pack8(q0);
      *reinterpret_cast<uint4*>(a.Qc + orow + c0 + half) = pack8(q1);
    }
    if (n_sink > 0) {
      const int64_t zrow = (((int64_t)b * a.Hq + h) * a.T + i) * n_sink;
      for (int j = 0; j < n_sink; ++j) {
        // every thread of a row group takes the same branch (same i and j)
        float z = -CUDART_INF_F;
        if (j <= i) {
          const bool capped = a.L > 0 && (i - j) > a.L;
          float acc = 0.f;
          if (sinks_in_smem) {
            const float* kv = capped ? s_sink_raw[j] : s_sink_rot[j];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              acc = fmaf(capped ? q0[e] : r0[e], kv[c0 + e], acc);
              acc = fmaf(capped ? q1[e] : r1[e], kv[c0 + e + half], acc);
            }
          } else {
            const __nv_bfloat16* kp = K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st;
            float k0[8], k1[8], kc[8], ks[8];
            unpack8(*reinterpret_cast<const uint4*>(kp + c0), k0);
            unpack8(*reinterpret_cast<const uint4*>(kp + c0 + half), k1);
            load_tab8(a.tab, j, half, c0, kc, ks);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              if (capped) {
                acc = fmaf(q0[e], k0[e], fmaf(q1[e], k1[e], acc));
              } else {
                acc = fmaf(r0[e], k0[e] * kc[e] - k1[e] * ks[e], acc);
                acc = fmaf(r1[e], k1[e] * kc[e] + k0[e] * ks[e], acc);
              }
            }
          }
          for (int o = tpr / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(grp_mask, acc, o);
          z = acc;
        }
        if (sub == (j % tpr)) a.sink_z[zrow + j] = z;
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
  if (a.d != 64 && a.d != 128) return cudaErrorInvalidValue;
  if (a.B == 0 || a.T == 0) return cudaSuccess;
  dim3 grid((a.T + kRowsPerBlock - 1) / kRowsPerBlock, std::max(a.Hq, a.Hkv), 2 * a.B);
  prep_kernel<<<grid, kPrepThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace sattn
