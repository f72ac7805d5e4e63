// segment.cu -- K7: retrieval for segmented execution.
//
// "Training-Inference Consistent Segmented Execution for Long-Context LLMs"
// (sections 整体框架 and 关键设计): before segment s, each long head takes
// the top-k from a detached, read-only pool of earlier keys using the
// segment-end query, and prepends the retrieved R keys as a prefix at
// positions 0..P-1 while the segment moves to P + t.
//
// Reading used here (the pages leave the score open): the pool is every key
// j < sS of the head's kv head, unrotated; it is cut into blocks of
// `blk` keys; a block scores max_{j in block} <q_{sS-1}, k_j> with the
// unrotated query of the previous segment's last token; the best R/blk
// blocks are taken (ties to the lower block) and laid out in ascending
// block order.
//
// Rotary re-basing: only distances enter a rotary logit, so the segment's
// queries and keys keep their global positions and each prefix key p is
// rotated to the virtual position sS - P + p, which puts it at distance
// P + t - p from the query at sS + t, exactly as positions p and P + t do.
//
// Three kernels:
//  1. block_score_kernel: every key of the largest pool is read once and
//     dotted with up to 16 segment-end queries at a time (fp32, queries held
//     in registers, a key spread over d/8 lanes with 16-byte loads); the
//     per-key dots go through shared memory into per-block maxima;
//  2. block_select_kernel: per (segment, long head) a bitonic sort of the
//     pool's block scores by (score desc, block asc), the first R/blk kept
//     and put in ascending block order;
//  3. prefix_assemble_kernel: gathers the chosen K rows (rotated to their
//     virtual positions) and V rows into the dense prefix planes the
//     attention kernel loads by TMA.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "simt.cuh"

namespace sattn {

namespace {

constexpr int kThreads = 256;
constexpr int kChunkKeys = 128;  // keys scored per pass of a CTA
constexpr int kQG = 16;          // segment-end queries per pass

// index of segment s in the per-segment arrays, and their count
__device__ __forceinline__ size_t seg_at(const SegRetrArgs& a, int s) { return (size_t)(s - a.s_base); }
__device__ __forceinline__ size_t seg_n(const SegRetrArgs& a) { return (size_t)(a.N - a.s_base); }

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 v = __bfloat1622float2(h[e]);
    f[2 * e] = v.x;
    f[2 * e + 1] = v.y;
  }
}

// grid (ceil(nblk_pool / nblk_cta), n_long, B).  CTA x scores blocks
// [x * nblk_cta, ...) of the pool of its long head for every segment s >= s_lo:
// score[b, slot, s, u] = max over the block's keys of <q_{sS-1}, k_j>.
// Entries whose block lies beyond segment s's pool are written too and
// never read.
template <int D>
__global__ void __launch_bounds__(kThreads) block_score_kernel(SegRetrArgs a, int nblk_pool, int nblk_cta) {
  constexpr int LPK = D / 8;     // lanes per key, 8 elements each
  constexpr int KPW = 32 / LPK;  // keys per warp per step
  __shared__ float sdot[kChunkKeys][kQG + 1];
  __shared__ float smax[kChunkKeys][kQG];  // per block of this CTA (nblk_cta <= kChunkKeys)
  const int slot = blockIdx.y, b = blockIdx.z;
  const int h = a.long_heads[slot];
  const int g = h / (a.Hq / a.Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPK;
  const int u0 = blockIdx.x * nblk_cta;
  const int u1 = min(u0 + nblk_cta, nblk_pool);
  const int k_begin = u0 * a.blk, k_end = u1 * a.blk;
  const __nv_bfloat16* kb = a.K + b * a.k_sb + g * a.k_sh;
  const __nv_bfloat16* qb = a.q_end ? nullptr : a.Q + b * a.q_sb + h * a.q_sh;
  for (int s0 = a.s_lo; s0 < a.N; s0 += kQG) {
    // this lane's 8 elements of the (up to) 16 segment-end queries
    float qr[kQG][8];
#pragma unroll
    for (int q = 0; q < kQG; ++q) {
      const int s = s0 + q;
      if (s < a.N) {
        const __nv_bfloat16* qe = a.q_end ? a.q_end + b * a.qe_sb + h * a.qe_sh
                                          : qb + (int64_t)(s * a.S - 1) * a.q_st;
        unpack8(*reinterpret_cast<const uint4*>(qe + sub * 8), qr[q]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) qr[q][e] = 0.f;
      }
    }
    for (int x = threadIdx.x; x < (u1 - u0) * kQG; x += kThreads) smax[x / kQG][x % kQG] = -CUDART_INF_F;
    for (int c0 = k_begin; c0 < k_end; c0 += kChunkKeys) {
      // every key load of this warp's share of the chunk is issued before the
      // first dot product (kSteps 16-byte loads in flight per lane)
      constexpr int kStep = (kThreads / 32) * KPW;  // keys per step of the whole CTA
      constexpr int kSteps = kChunkKeys / kStep;
      uint4 raw[kSteps];
#pragma unroll
      for (int u = 0; u < kSteps; ++u) {
        const int j = c0 + u * kStep + warp * KPW + lane / LPK;
        raw[u] = (j < k_end) ? *reinterpret_cast<const uint4*>(kb + (int64_t)j * a.k_st + sub * 8)
                             : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kSteps; ++u) {
        const int kk = u * kStep + warp * KPW + lane / LPK;
        const int j = c0 + kk;
        float kv[8];
        unpack8(raw[u], kv);  // keys past the end carry zeros
        float dot[kQG];
#pragma unroll
        for (int q = 0; q < kQG; ++q) {
          float A0 = 0.f, A1 = 0.f;
#pragma unroll
          for (int e = 0; e < 8; e += 2) fma2(A0, A1, qr[q][e], qr[q][e + 1], kv[e], kv[e + 1], A0, A1);
          dot[q] = A0 + A1;
        }
        // the whole warp takes part
        group_reduce_transposed<kQG, LPK>(dot, 0xffffffffu, lane);
        constexpr int per = kQG >= LPK ? kQG / LPK : 1;
        constexpr int dup = kQG >= LPK ? 1 : LPK / kQG;
        if (j < k_end && sub % dup == 0) {
#pragma unroll
          for (int q = 0; q < per; ++q) sdot[kk][(sub / dup) * per + q] = dot[q];
        }
      }
      __syncthreads();
      // block maxima of this chunk: a warp per (block, query)
      const int c1 = min(c0 + kChunkKeys, k_end);
      for (int pr = warp; pr < (u1 - u0) * kQG; pr += kThreads / 32) {
        const int bl = pr / kQG, q = pr % kQG;
        const int lo = max((u0 + bl) * a.blk, c0), hi = min((u0 + bl + 1) * a.blk, c1);
        float m = -CUDART_INF_F;
        for (int j = lo + lane; j < hi; j += 32) m = fmaxf(m, sdot[j - c0][q]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) smax[bl][q] = fmaxf(smax[bl][q], m);
      }
      __syncthreads();
    }
    const int nblk_all = a.T / a.blk;
    for (int x = threadIdx.x; x < (u1 - u0) * kQG; x += kThreads) {
      const int bl = x / kQG, q = x % kQG;
      const int s = s0 + q;
      if (s < a.N) a.score[(((size_t)b * a.n_long + slot) * seg_n(a) + seg_at(a, s)) * nblk_all + u0 + bl] = smax[bl][q];
    }
    __syncthreads();
  }
}

// total order key for a descending sort: larger score first, then the lower block
__device__ __forceinline__ unsigned long long order_key(float z, int u) {
  const uint32_t bits = __float_as_uint(z);
  const uint32_t ord = (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);  // monotone in z
  return ((unsigned long long)ord << 32) | (0xFFFFFFFFu - (uint32_t)u);
}

// grid (N - s_lo, n_long, B): segment s = blockIdx.x + s_lo.  Dynamic
// shared memory: next_pow2(blocks of the largest pool) 64-bit keys.
__global__ void __launch_bounds__(kThreads) block_select_kernel(SegRetrArgs a) {
  extern __shared__ unsigned long long keys[];
  __shared__ int chosen[1024];
  const int s = blockIdx.x + a.s_lo;
  const int slot = blockIdx.y;
  const int b = blockIdx.z;
  const int h = a.long_heads[slot];
  const int nb = a.R / a.blk;
  const int nblocks = s * a.S / a.blk;
  const int nsel = min(nb, nblocks);
  int P2 = 1;
  while (P2 < nblocks) P2 <<= 1;
  const int nblk_all = a.T / a.blk;
  const float* score = a.score + (((size_t)b * a.n_long + slot) * seg_n(a) + seg_at(a, s)) * nblk_all;
  for (int u = threadIdx.x; u < P2; u += kThreads) keys[u] = (u < nblocks) ? order_key(score[u], u) : 0ull;
  __syncthreads();
  // bitonic sort, descending
  for (int k = 2; k <= P2; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int x = threadIdx.x; x < P2; x += kThreads) {
        const int y = x ^ jj;
        if (y > x) {
          const unsigned long long p = keys[x], q = keys[y];
          const bool first_half = (x & k) == 0;
          if (first_half ? (p < q) : (p > q)) {
            keys[x] = q;
            keys[y] = p;
          }
        }
      }
      __syncthreads();
    }
  }
  // the first nsel blocks, in ascending block order (rank by count)
  for (int x = threadIdx.x; x < nsel; x += kThreads) {
    const int u = (int)(0xFFFFFFFFu - (uint32_t)(keys[x] & 0xFFFFFFFFull));
    int rank = 0;
    for (int y = 0; y < nsel; ++y) {
      const int v = (int)(0xFFFFFFFFu - (uint32_t)(keys[y] & 0xFFFFFFFFull));
      rank += (v < u) ? 1 : 0;
    }
    chosen[rank] = u;
  }
  __syncthreads();
  if (threadIdx.x == 0) a.prefix_cnt[((size_t)b * a.n_long + slot) * seg_n(a) + seg_at(a, s)] = nsel * a.blk;
  int32_t* out = a.prefix_blocks + (((size_t)b * a.Hq + h) * seg_n(a) + seg_at(a, s)) * nb;
  for (int x = threadIdx.x; x < nb; x += kThreads) out[x] = x < nsel ? chosen[x] : -1;
}

// grid (Rpad / 8, (N - s_lo) * n_long, B); one warp per prefix row.  Lanes
// [0, d/8) rotate 4 pairs of K each (8-byte loads from both halves, the
// virtual position's cos/sin as two float4), lanes [16, 16 + d/8) copy 16
// bytes of V each.
template <int D>
__global__ void prefix_assemble_kernel(SegRetrArgs a, int Rpad) {
  constexpr int half = D / 2;
  constexpr int kLanes = D / 8;  // K lanes (4 pairs each) = V lanes (16 bytes each)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = blockIdx.x * 8 + warp;
  const int s = blockIdx.y % (a.N - a.s_lo) + a.s_lo;
  const int slot = blockIdx.y / (a.N - a.s_lo);
  const int b = blockIdx.z;
  if (p >= Rpad) return;
  const int h = a.long_heads[slot];
  const int g = h / (a.Hq / a.Hkv);
  const int cnt = a.prefix_cnt[((size_t)b * a.n_long + slot) * seg_n(a) + seg_at(a, s)];
  const size_t orow = ((((size_t)b * a.n_long + slot) * seg_n(a) + seg_at(a, s)) * Rpad + p) * D;
  if (p >= cnt) {
    if (lane < kLanes) {
      reinterpret_cast<uint4*>(a.Kpre + orow)[lane] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(a.Vpre + orow)[lane] = make_uint4(0, 0, 0, 0);
    }
    return;
  }
  const int nb = a.R / a.blk;
  const int blk_id = a.prefix_blocks[(((size_t)b * a.Hq + h) * seg_n(a) + seg_at(a, s)) * nb + p / a.blk];
  const int j = blk_id * a.blk + p % a.blk;
  const int vpos = s * a.S - cnt + p;
  if (lane < kLanes) {
    const int c = lane * 4;
    const __nv_bfloat16* kp = a.K + b * a.k_sb + g * a.k_sh + (int64_t)j * a.k_st;
    const uint2 lo = *reinterpret_cast<const uint2*>(kp + c);
    const uint2 hi = *reinterpret_cast<const uint2*>(kp + c + half);
    const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&lo);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hi);
    float k0[4], k1[4], cs[4], sn[4];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float2 x = __bfloat1622float2(l2[e]), y = __bfloat1622float2(h2[e]);
      k0[2 * e] = x.x;
      k0[2 * e + 1] = x.y;
      k1[2 * e] = y.x;
      k1[2 * e + 1] = y.y;
    }
    if (a.tab) {
      const float4* t = reinterpret_cast<const float4*>(a.tab + (int64_t)vpos * half + c);
      const float4 t0 = t[0], t1 = t[1];
      cs[0] = t0.x; sn[0] = t0.y; cs[1] = t0.z; sn[1] = t0.w;
      cs[2] = t1.x; sn[2] = t1.y; cs[3] = t1.z; sn[3] = t1.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        cs[e] = 1.f;
        sn[e] = 0.f;
      }
    }
    uint2 olo, ohi;
    __nv_bfloat162* o_l = reinterpret_cast<__nv_bfloat162*>(&olo);
    __nv_bfloat162* o_h = reinterpret_cast<__nv_bfloat162*>(&ohi);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      o_l[e] = __floats2bfloat162_rn(k0[2 * e] * cs[2 * e] - k1[2 * e] * sn[2 * e],
                                     k0[2 * e + 1] * cs[2 * e + 1] - k1[2 * e + 1] * sn[2 * e + 1]);
      o_h[e] = __floats2bfloat162_rn(k1[2 * e] * cs[2 * e] + k0[2 * e] * sn[2 * e],
                                     k1[2 * e + 1] * cs[2 * e + 1] + k0[2 * e + 1] * sn[2 * e + 1]);
    }
    *reinterpret_cast<uint2*>(a.Kpre + orow + c) = olo;
    *reinterpret_cast<uint2*>(a.Kpre + orow + c + half) = ohi;
  } else if (lane >= 16 && lane < 16 + kLanes) {
    const __nv_bfloat16* vp = a.V + b * a.v_sb + g * a.v_sh + (int64_t)j * a.v_st;
    reinterpret_cast<uint4*>(a.Vpre + orow)[lane - 16] = reinterpret_cast<const uint4*>(vp)[lane - 16];
  }
}

template <int D>
cudaError_t launch_d(const SegRetrArgs& a, cudaStream_t st) {
  const int nblk_pool = (a.N - 1) * a.S / a.blk;  // blocks of the largest pool
  if (nblk_pool > 0) {
    const int nblk_cta = std::max(1, kChunkKeys / a.blk);
    dim3 g1((nblk_pool + nblk_cta - 1) / nblk_cta, a.n_long, a.B);
    block_score_kernel<D><<<g1, kThreads, 0, st>>>(a, nblk_pool, nblk_cta);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  int P2 = 1;
  while (P2 < nblk_pool) P2 <<= 1;
  const size_t smem = (size_t)P2 * sizeof(unsigned long long);
  cudaError_t e = cudaFuncSetAttribute(block_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 g2(a.N - a.s_lo, a.n_long, a.B);
  block_select_kernel<<<g2, kThreads, smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int Rpad = (a.R + kTile - 1) / kTile * kTile;
  dim3 g3(Rpad / 8, (a.N - a.s_lo) * a.n_long, a.B);
  prefix_assemble_kernel<D><<<g3, 256, 0, st>>>(a, Rpad);
  return cudaGetLastError();
}

}  // namespace

size_t segment_score_bytes(int B, int n_long, int N, int T, int blk) {
  return (size_t)B * n_long * N * (size_t)(T / blk) * sizeof(float);
}

bool segment_retrieval_supported(int T, int S, int blk) {
  const int nblk_pool = (T / S - 1) * S / blk;
  int P2 = 1;
  while (P2 < nblk_pool) P2 <<= 1;
  return (size_t)P2 * sizeof(unsigned long long) <= kSegSelectSmemMax;
}

cudaError_t launch_segment_retrieval(const SegRetrArgs& a, cudaStream_t st) {
  if (a.s_lo < 1 || a.s_base < 0 || a.s_base > a.s_lo) return cudaErrorInvalidValue;
  if (a.N <= a.s_lo || a.n_long == 0 || a.R == 0 || a.B == 0) return cudaSuccess;
  if (a.d == 128) return launch_d<128>(a, st);
  if (a.d == 64) return launch_d<64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace sattn
