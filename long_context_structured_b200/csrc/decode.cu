// decode.cu -- one decoding step: the newest token's query over the
// structured key set of its position.
//
// For the query at position i = T - 1 (its own key and value are the last
// cache entry) the kept keys are the same disjoint parts as in prefill
// ("LM-Infinite", section 方法: the starting span and the recent window;
// "SepLLM", section 五.2: every earlier separator): sinks j < n_start,
// window max(n_start, i - w) <= j <= i, separators n_start <= j < i - w.
// A key farther than L_pretrain takes the capped logit <R(L) q, k_j> with
// the unrotated key, the others <R(i) q, R(j) k_j>.
//
// Split-K over the kept keys (memory-bound: each kept K and V row is read
// once): a CTA takes a chunk of kChunk kept keys of one (batch, kv head) for
// all query heads of that kv head's group.  It first stages all the chunk's
// K and V rows in shared memory (64 KB at d = 128, so that every byte the
// CTA needs is in flight at once: one bulk copy per tensor for a run of
// consecutive rows, else 16-byte asynchronous copies), then computes the
// logits from the staged K rows (a key's head dimension spread over a few
// lanes, each holding some rotary pairs and their partners c + d/2), then,
// with the chunk's per-head maximum known, the weighted V rows.  The chunk's
// (max, sum, unnormalised O) per head go to the workspace; a merge kernel,
// launched as the split-K kernel's programmatic dependent, combines them
// into O and LSE.
//
// The rotations are computed in the kernel, not read from a table: the
// angle of a position in turns from a two-float turn rate, reduced by whole
// turns in fp32 without rounding loss, then the hardware sine and cosine;
// along a run of consecutive positions a lane steps its query's (or its
// keys') rotation by one fixed rotation (angle addition in fp32) instead.
#include <algorithm>
#include <cmath>

#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "select.cuh"
#include "simt.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

constexpr int kThreads = 128;  // top-k logit kernel: 4 warps
constexpr int kChunk = 128;    // kept keys per CTA
static_assert(kThreads >= kChunk, "a thread looks up one slot's key position");
// split-K kernel: 8 warps (two CTAs per SM) with one or two query heads per
// kv head, 4 warps (three CTAs per SM, by shared memory) with more, whose
// per-lane query state needs the registers
template <int REP>
struct PartCfg {
  static constexpr int NT = REP <= 2 ? 256 : 128;
  static constexpr int MIN_BLOCKS = REP <= 2 ? 2 : 3;
};
constexpr int kMaxChunks = 4096;  // chunks one step may merge (keys up to 4096 * kChunk)

// programmatic dependent launch: let the next kernel of the step start its
// independent work early / wait for the previous kernel's results
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// 16-byte asynchronous copy global -> shared; `valid` false fills zeros
// without reading the source
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// one bulk copy (the copy engine) of `bytes` contiguous bytes global ->
// shared, completing on the mbarrier's transaction count; no multicast
__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// wait sites reported in the status word
constexpr int kSiteDecodeK = 101, kSiteDecodeV = 102, kSiteTopkK = 103;

// Staging of a chunk's rows: one bulk copy per tensor when the rows are
// consecutive in memory (bars[t] completes when they land), else 16-byte
// asynchronous copies per piece (tensor t is copy group t).
struct StageWait {
  bool bulk;
  uint64_t* bars;
  volatile int* abort_flag;
  int32_t* status;
  // wait for tensor t (0: first, 1: second) of a two-tensor staging, or the
  // only tensor of a one-tensor staging (ntensors 1); true when it landed.
  // Every thread of the block calls it; the result is uniform.
  __device__ __forceinline__ bool wait(int t, int ntensors, int site) {
    if (bulk) {
      // one thread polls; the others wait at the barrier without issuing
      if (threadIdx.x == 0) mbar_wait(bars + t, 0, abort_flag, status, site);
    } else if (ntensors == 2 && t == 0) {
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    return *abort_flag == 0;
  }
  // after a failed wait: give the copies still in flight a bounded time to land
  __device__ __forceinline__ void drain(int ntensors) {
    if (!bulk || threadIdx.x != 0) return;
    for (int t = 0; t < ntensors; ++t) {
      const uint32_t a = smem_u32(bars + t);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
      }
    }
  }
};

// zero 16-byte pieces [from, to) of a shared array (rows past a chunk's end
// when the chunk was bulk-copied)
__device__ __forceinline__ void zero_pieces(void* base, int from, int to, int nthreads) {
  uint4* p = reinterpret_cast<uint4*>(base);
  for (int x = from + (int)threadIdx.x; x < to; x += nthreads) p[x] = make_uint4(0u, 0u, 0u, 0u);
}

struct KeySet {
  int n_sink, win_lo, n_win, n_sep;
  __device__ __forceinline__ int n() const { return n_sink + n_win + n_sep; }
};

// cache length of sequence b: the per-sequence length when given (a
// streaming cache), else T
__device__ __forceinline__ int cache_len(const DecodeArgs& a, int b) { return a.seq_len ? a.seq_len[b] : a.T; }

__device__ __forceinline__ KeySet key_set(const DecodeArgs& a, int b) {
  KeySet s;
  const int Tb = cache_len(a, b);
  const int i = Tb - 1;
  s.n_sink = min(a.n_start, Tb);
  s.win_lo = max(s.n_sink, i - a.window);
  s.n_win = max(0, i - s.win_lo + 1);
  const int thr = i - a.window;  // separators kept: n_start <= j < i - w
  s.n_sep = (a.sep_words && thr > 0) ? sep_before(a.sep_words, a.T, b, thr) : 0;
  return s;
}

__device__ __forceinline__ int key_at(const DecodeArgs& a, const KeySet& s, int b, int e) {
  if (e < s.n_sink) return e;
  e -= s.n_sink;
  if (e < s.n_win) return s.win_lo + e;
  return a.sep_pos[(size_t)b * a.T + (e - s.n_win)];
}

// ---- packed fp32 pairs (one f32x2 instruction per two lanes of work) ----
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// two bf16 (one 32-bit word, low half first) as a float pair
__device__ __forceinline__ float2 bf2f(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// EPL consecutive bf16 (16, 8 or 4 bytes) as EPL / 2 float pairs
template <int H>
__device__ __forceinline__ void load_pairs(const __nv_bfloat16* p, float2 (&out)[H]) {
  if constexpr (H == 4) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    out[0] = bf2f(u.x);
    out[1] = bf2f(u.y);
    out[2] = bf2f(u.z);
    out[3] = bf2f(u.w);
  } else if constexpr (H == 2) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    out[0] = bf2f(u.x);
    out[1] = bf2f(u.y);
  } else {
    out[0] = bf2f(*reinterpret_cast<const uint32_t*>(p));
  }
}

// (cos, sin) of rotary pair c at position p.  The angle in turns, p f_c
// with f_c = s theta^(-2c/d) / (2 pi) split on the host into fp32 parts
// hi + lo: p * hi is formed with its exact rounding residual (one fma), its
// whole turns removed exactly, and p * lo added, which leaves the reduced
// angle to about 3e-8 turns for the positions a step uses (below 2^19);
// then the hardware sine and cosine of that angle, within 1.02 pi of zero
// (absolute error about 2^-21).
// The per-pair rotation constants, copied once per CTA from the kernel
// parameters into shared memory (lanes index them by pair, which a
// parameter-space load would serialise).
struct RopeTab {
  float hi[64], lo[64];  // turns per position, hi + lo
  float2 st[64];         // (cos, sin) of the rotation by KPS positions
};

__device__ __forceinline__ void load_rope_tab(const DecodeArgs& a, RopeTab& t, int half) {
  const int x = threadIdx.x;
  if (x < half) {
    t.hi[x] = a.turn_hi[x];
    t.lo[x] = a.turn_lo[x];
    t.st[x] = a.step_cs[x];
  }
}

// |p| < 2^22 and |t1| < 2^22: the int-to-float conversion and the rounding
// to a whole number of turns are done by adding 1.5 * 2^23 (exact at that
// magnitude), which keeps them off the conversion unit.
__device__ __forceinline__ float2 rope_cs(const RopeTab& t, int p, int c) {
  constexpr float kMagic = 12582912.f;  // 1.5 * 2^23
  const float fp = __int_as_float(0x4B400000 + p) - kMagic;
  const float hi = t.hi[c];
  const float t1 = fp * hi;
  const float e1 = fmaf(fp, hi, -t1);
  const float whole = __fsub_rn(__fadd_rn(t1, kMagic), kMagic);
  const float r = (t1 - whole) + fmaf(fp, t.lo[c], e1);
  float s, co;
  __sincosf(r * 6.283185307179586f, &s, &co);
  return make_float2(co, s);
}

// A lane's rotation for its EPL = 2H pairs [p0, p0 + EPL): cosines C[h] and
// sines S[h] of pairs (p0 + 2h, p0 + 2h + 1).
template <int H>
struct Rot {
  float2 C[H], S[H];
};

template <int H>
__device__ __forceinline__ Rot<H> rope_rot(const DecodeArgs& a, const RopeTab& rt, int p, int p0) {
  Rot<H> t;
#pragma unroll
  for (int h = 0; h < H; ++h) {
    float2 u = make_float2(1.f, 0.f), v = make_float2(1.f, 0.f);
    if (a.rope) {
      u = rope_cs(rt, p, p0 + 2 * h);
      v = rope_cs(rt, p, p0 + 2 * h + 1);
    }
    t.C[h] = make_float2(u.x, v.x);
    t.S[h] = make_float2(u.y, v.y);
  }
  return t;
}

// (x0, x1) <- R (x0, x1) per pair: x0 c - x1 s, x1 c + x0 s
template <int H>
__device__ __forceinline__ void rotate(float2 (&x0)[H], float2 (&x1)[H], const Rot<H>& t) {
#pragma unroll
  for (int h = 0; h < H; ++h) {
    const float2 y0 = fsub2(fmul2(x0[h], t.C[h]), fmul2(x1[h], t.S[h]));
    const float2 y1 = ffma2(x0[h], t.S[h], fmul2(x1[h], t.C[h]));
    x0[h] = y0;
    x1[h] = y1;
  }
}

// t <- t composed with the rotation (sc, ss) (angle addition), nss = -ss
template <int H>
__device__ __forceinline__ void rot_advance(Rot<H>& t, const Rot<H>& st, const float2 (&nss)[H]) {
#pragma unroll
  for (int h = 0; h < H; ++h) {
    const float2 c = ffma2(t.S[h], nss[h], fmul2(t.C[h], st.C[h]));
    const float2 s = ffma2(t.C[h], st.S[h], fmul2(t.S[h], st.C[h]));
    t.C[h] = c;
    t.S[h] = s;
  }
}

// Lane layout of the logit pass.  A key is spread over LPK lanes (8, or 16
// for eight query heads per kv head), each holding EPL rotary pairs (16 or 8
// elements of the row) as H = EPL / 2 float pairs, so a warp works on KPS =
// 32 / LPK keys at once with 16-byte shared-memory loads; KPW key slots per
// warp, KPL keys per lane (a lane's keys are the warp's slots kg, kg + KPS,
// ...).  A lane accumulates the partial dot products of NB keys for all REP
// heads (NB * REP = LPK values) before one transposed reduction over the
// key's lanes hands each lane one finished logit.
template <int D, int REP, int NW = kThreads / 32>
struct Tiling {
  static constexpr int half = D / 2;
  static constexpr int LPK = (REP >= 8) ? 16 : 8;       // lanes per key
  static constexpr int KPS = 32 / LPK;                  // keys per warp step
  static constexpr int EPL = half / LPK;                // rotary pairs per lane
  static constexpr int H = EPL / 2;                     // float pairs per half row
  static constexpr int KPW = kChunk / NW;              // keys per warp
  static constexpr int KPL = KPW / KPS;                 // keys per lane
  static constexpr int NB = (LPK / REP < KPL) ? LPK / REP : KPL;  // keys per reduction
  static constexpr int NV = NB * REP;                   // values per reduction (<= LPK)
  static constexpr int UNR = (REP >= 4) ? 1 : 2;        // pass 2: key steps loaded together
  static_assert(REP <= LPK && KPL % NB == 0 && KPW % (KPS * UNR) == 0 && (EPL == 8 || EPL == 4 || EPL == 2),
                "decode tiling");
};

// This lane's raw query pairs of each head of kv group g: first-half
// elements p0 .. p0 + EPL - 1 in q0, their partners in q1.
template <int D, int REP>
__device__ __forceinline__ void load_query(const DecodeArgs& a, int b, int g, int p0,
                                           float2 (&q0)[REP][Tiling<D, REP>::H],
                                           float2 (&q1)[REP][Tiling<D, REP>::H]) {
  constexpr int half = D / 2, H = Tiling<D, REP>::H;
#pragma unroll
  for (int r = 0; r < REP; ++r) {
    const __nv_bfloat16* qp = a.Q + (size_t)b * a.q_sb + (size_t)(g * REP + r) * a.q_sh;
    load_pairs<H>(qp + p0, q0[r]);
    load_pairs<H>(qp + p0 + half, q1[r]);
  }
}

// Stage the CTA's kChunk rows of one kv head's cache into dst[slot * D ..]:
// row `slot` is position key(slot), or zeros when key(slot) < 0.  16-byte
// pieces; a thread keeps one piece column, consecutive threads take
// consecutive pieces of a row.
template <int D, int NT, class Key>
__device__ __forceinline__ void stage_rows(__nv_bfloat16* dst, const __nv_bfloat16* base, int64_t st, Key key) {
  constexpr int PR = D / 8;       // pieces per row
  constexpr int RPP = NT / PR;    // rows per pass
  const int c = (int)threadIdx.x % PR;
#pragma unroll
  for (int slot = (int)threadIdx.x / PR; slot < kChunk; slot += RPP) {
    const int j = key(slot);
    cp_async16(dst + slot * D + c * 8, base + (int64_t)(j < 0 ? 0 : j) * st + c * 8, j >= 0);
  }
}

// How the logit pass pairs a staged raw key k_j with the query q (position i):
//   kRotNone: as they are (no rotation; or every key of the warp lies past
//             the cap and the query is rotated to L: <R(L) q, k_j>);
//   kRotRun:  the warp's slots hold consecutive positions run_j0, run_j0 + 1,
//             ...: <R(i) q, R(j) k_j> = <R(i - j) q, k_j>.  With one or two
//             query heads per kv head the lane's rotated queries are
//             stepped by R(-KPS) from key to key; with more, the key's
//             rotation R(j) is stepped by R(KPS) and applied to the key;
//   kRotEach: each key's rotation R(j) computed from its position.
// A key past the cap (i - j > L) takes <R(L) q, k_j> in every mode.
enum { kRotNone = 0, kRotRun = 1, kRotEach = 2 };

// The logit pass over one warp's KPW staged key slots [w_lo, w_lo + KPW)
// (sK: the chunk's K rows, raw) against the lane's raw query pairs q0 / q1:
// per lane NB keys' partial dot products for every head, then one
// transposed butterfly over the key's lanes, after which lane sub holds the
// logit of key sub / REP of the batch for head sub % REP.  key_of(slot)
// gives the slot's key position (-1: none); emit(r, slot, j, dot) receives
// head r's unscaled logit, once per (key, head).  mode kRotNone with
// none_pos >= 0 rotates the query to none_pos first.
template <int D, int REP, int NW, class KeyOf, class Emit>
__device__ __forceinline__ void logits_pass(const DecodeArgs& a, const RopeTab& rt, int i, const __nv_bfloat16* sK,
                                            int w_lo, int mode,
                                            int run_j0, int none_pos, int lane,
                                            const float2 (&qr0)[REP][Tiling<D, REP>::H],
                                            const float2 (&qr1)[REP][Tiling<D, REP>::H], KeyOf key_of,
                                            Emit emit) {
  using TL = Tiling<D, REP, NW>;
  constexpr int half = D / 2, LPK = TL::LPK, KPS = TL::KPS, EPL = TL::EPL, H = TL::H, KPL = TL::KPL, NB = TL::NB,
                NV = TL::NV;
  constexpr bool kStepQuery = REP <= 2;  // run mode: step the query rotation, not the key's
  const int sub = lane % LPK, kg = lane / LPK;
  const int p0 = sub * EPL;
  const bool need_cap = mode != kRotNone && a.L > 0 && i > a.L && (mode == kRotEach || run_j0 < i - a.L);
  // q: the query the keys are dotted with (rotated per mode); qc: rotated to L
  float2 q0[REP][H], q1[REP][H], qc0[REP][H], qc1[REP][H];
  auto rotated = [&](int pos, float2 (&y0)[REP][H], float2 (&y1)[REP][H]) {
    const Rot<H> t = rope_rot<H>(a, rt, pos, p0);
#pragma unroll
    for (int r = 0; r < REP; ++r) {
#pragma unroll
      for (int h = 0; h < H; ++h) {
        y0[r][h] = qr0[r][h];
        y1[r][h] = qr1[r][h];
      }
      rotate<H>(y0[r], y1[r], t);
    }
  };
  const bool step_q = mode == kRotRun && kStepQuery;
  if (mode == kRotNone) {
    if (none_pos >= 0) rotated(none_pos, q0, q1);
    else {
#pragma unroll
      for (int r = 0; r < REP; ++r)
#pragma unroll
        for (int h = 0; h < H; ++h) {
          q0[r][h] = qr0[r][h];
          q1[r][h] = qr1[r][h];
        }
    }
  } else if (step_q) {
    rotated(i - (run_j0 + kg), q0, q1);  // R(i - j) q for the lane's first key
    if (need_cap) rotated(a.L, qc0, qc1);
  } else {
    rotated(i, q0, q1);
  }
  // run stepping: (sc, ss) the rotation by KPS positions, nss = -ss
  Rot<H> st, cur, cap;
  float2 nss[H];
  if (mode == kRotRun) {
#pragma unroll
    for (int h = 0; h < H; ++h) {
      const float2 u = rt.st[p0 + 2 * h], v = rt.st[p0 + 2 * h + 1];
      st.C[h] = make_float2(u.x, v.x);
      st.S[h] = make_float2(u.y, v.y);
      nss[h] = make_float2(-u.y, -v.y);
    }
    if (!kStepQuery) cur = rope_rot<H>(a, rt, run_j0 + kg, p0);
  }
  if (need_cap && !step_q) cap = rope_rot<H>(a, rt, i - a.L, p0);
#pragma unroll 1
  for (int m0 = 0; m0 < KPL; m0 += NB) {
    float2 acc[NV];  // [NB keys][REP heads], pairwise partial sums
#pragma unroll
    for (int x = 0; x < NV; ++x) acc[x] = make_float2(0.f, 0.f);
#pragma unroll
    for (int kb = 0; kb < NB; ++kb) {
      const int el = w_lo + kg + KPS * (m0 + kb);
      float2 k0[H], k1[H];
      load_pairs<H>(sK + el * D + p0, k0);
      load_pairs<H>(sK + el * D + p0 + half, k1);
      const int j = (mode == kRotRun) ? run_j0 + (el - w_lo) : key_of(el);
      const bool capped = need_cap && i - j > a.L;
      if (step_q) {
        // keys past the cap pair with R(L) q, the others with R(i - j) q
#pragma unroll
        for (int r = 0; r < REP; ++r)
#pragma unroll
          for (int h = 0; h < H; ++h) {
            const float2 x0 = capped ? qc0[r][h] : q0[r][h], x1 = capped ? qc1[r][h] : q1[r][h];
            acc[kb * REP + r] = ffma2(x0, k0[h], ffma2(x1, k1[h], acc[kb * REP + r]));
          }
        // R(i - j - KPS) q = R(-KPS) R(i - j) q: rotate by (sc, -ss)
#pragma unroll
        for (int r = 0; r < REP; ++r)
#pragma unroll
          for (int h = 0; h < H; ++h) {
            const float2 y0 = ffma2(q1[r][h], st.S[h], fmul2(q0[r][h], st.C[h]));
            const float2 y1 = ffma2(q0[r][h], nss[h], fmul2(q1[r][h], st.C[h]));
            q0[r][h] = y0;
            q1[r][h] = y1;
          }
      } else {
        if (mode != kRotNone) {
          if (capped) {
            rotate<H>(k0, k1, cap);
          } else if (mode == kRotRun) {
            rotate<H>(k0, k1, cur);
          } else {
            rotate<H>(k0, k1, rope_rot<H>(a, rt, j < 0 ? 0 : j, p0));
          }
          if (mode == kRotRun) rot_advance<H>(cur, st, nss);
        }
#pragma unroll
        for (int r = 0; r < REP; ++r)
#pragma unroll
          for (int h = 0; h < H; ++h) acc[kb * REP + r] = ffma2(q0[r][h], k0[h], ffma2(q1[r][h], k1[h], acc[kb * REP + r]));
      }
    }
    float v[NV];
#pragma unroll
    for (int x = 0; x < NV; ++x) v[x] = acc[x].x + acc[x].y;
    group_reduce_transposed<NV, LPK>(v, 0xffffffffu, lane);
    // value sub / DUP (DUP lanes hold each)
    constexpr int DUP = LPK / NV;
    const int vi = sub / DUP;
    const int el = w_lo + kg + KPS * (m0 + vi / REP);
    if (sub % DUP == 0) emit(vi % REP, el, key_of(el), v[0]);
  }
}

// grid (B * Hkv, chunks): the (batch, kv head) index varies fastest, so the
// chunks that hold keys (the low ones) are dispatched before the empty ones.
// The chunk's K and V rows are copied to shared memory first (K and V as two
// copy groups); then (1) logits (logits_pass) to shared memory, (2) with the
// chunk's per-head maximum and the weights p = 2^(z - m) taken once per
// (key, head): O += p v.  No running rescale.  The chunk's partials go to
// the workspace for the merge kernel.
template <int D, int REP>
__global__ void __launch_bounds__(PartCfg<REP>::NT, PartCfg<REP>::MIN_BLOCKS) decode_partial_kernel(DecodeArgs a) {
  constexpr int kPartThreads = PartCfg<REP>::NT;
  constexpr int NW = kPartThreads / 32;
  using TL = Tiling<D, REP, NW>;
  constexpr int half = D / 2, LPK = TL::LPK, KPS = TL::KPS, EPL = TL::EPL, H = TL::H, KPW = TL::KPW, UNR = TL::UNR;
  extern __shared__ __align__(16) unsigned char dsm[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(dsm);  // [kChunk][D]
  __nv_bfloat16* sV = sK + kChunk * D;                         // [kChunk][D]
  float* red_o = reinterpret_cast<float*>(dsm);                // [warps][REP][D], over sK after pass 1
  static_assert(NW * REP * D * 4 <= kChunk * D * 2, "the O reduction fits over the K rows");
  __shared__ float s_p[REP][kChunk];  // logits, then weights
  __shared__ int s_j[kChunk];         // slot -> key position (-1: none)
  __shared__ float s_m[REP], s_l[REP];
  __shared__ RopeTab s_rt;
  __shared__ __align__(8) uint64_t s_bar[2];
  __shared__ int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPK, kg = lane / LPK;
  const int bg = blockIdx.x;
  const int g = bg % a.Hkv, b = bg / a.Hkv;
  grid_dep_launch();  // the merge kernel may be scheduled now; it waits for this grid
  // the key set of a cache with separators comes from the block map, the
  // previous kernel's output; without them it is a closed form, and the K
  // and V copies start before that kernel has finished
  if (a.sep_words) grid_dep_wait();
  const KeySet ks = key_set(a, b);
  const int n = ks.n();
  const int e_begin = blockIdx.y * kChunk;
  if (e_begin >= n) {  // this batch has fewer chunks
    grid_dep_wait();
    return;
  }
  const int n_here = min(n - e_begin, kChunk);
  const int i = cache_len(a, b) - 1;
  // a chunk inside the window holds consecutive positions: with contiguous
  // rows its K and V are one bulk copy each
  const bool bulk = e_begin >= ks.n_sink && e_begin + n_here <= ks.n_sink + ks.n_win && a.k_st == D && a.v_st == D;
  if (threadIdx.x == 0) {
    s_abort = 0;
    if (bulk) {
      mbar_init(&s_bar[0], 1);
      mbar_init(&s_bar[1], 1);
      fence_mbar_init();
    }
  }
  if (threadIdx.x < kChunk) s_j[threadIdx.x] = (int)threadIdx.x < n_here ? key_at(a, ks, b, e_begin + threadIdx.x) : -1;
  if (a.rope) load_rope_tab(a, s_rt, half);
  __syncthreads();
  const __nv_bfloat16* kb = a.K + (size_t)b * a.k_sb + (size_t)g * a.k_sh;
  const __nv_bfloat16* vb = a.V + (size_t)b * a.v_sb + (size_t)g * a.v_sh;
  if (bulk) {
    if (threadIdx.x == 0) {
      const size_t j0 = (size_t)(ks.win_lo + (e_begin - ks.n_sink));
      const uint32_t bytes = (uint32_t)n_here * D * 2;
      mbar_expect_tx(&s_bar[0], bytes);
      bulk_copy(sK, kb + j0 * D, bytes, &s_bar[0]);
      mbar_expect_tx(&s_bar[1], bytes);
      bulk_copy(sV, vb + j0 * D, bytes, &s_bar[1]);
    }
    zero_pieces(sK, n_here * D / 8, kChunk * D / 8, kPartThreads);
    zero_pieces(sV, n_here * D / 8, kChunk * D / 8, kPartThreads);
  } else {
    stage_rows<D, kPartThreads>(sK, kb, a.k_st, [&](int s) { return s_j[s]; });
    cp_async_commit();
    stage_rows<D, kPartThreads>(sV, vb, a.v_st, [&](int s) { return s_j[s]; });
    cp_async_commit();
  }
  StageWait sw{bulk, s_bar, &s_abort, a.status};
  grid_dep_wait();
  const int p0 = sub * EPL;  // this lane's pairs [p0, p0 + EPL)
  float2 q0[REP][H], q1[REP][H];
  load_query<D, REP>(a, b, g, p0, q0, q1);
  const float sl2 = a.scale_log2;
  const int w_lo = warp * KPW;
  // a warp whose keys all lie in the window holds consecutive positions
  const int e_w = e_begin + w_lo, e_w_end = min(e_w + KPW, n);
  const bool run = e_w >= ks.n_sink && e_w_end <= ks.n_sink + ks.n_win;
  if (!sw.wait(0, 2, kSiteDecodeK)) {
    sw.drain(2);
    return;
  }

  // ---- pass 1: logits ----
  const int mode = !a.rope ? kRotNone : (run ? kRotRun : kRotEach);
  logits_pass<D, REP, NW>(
      a, s_rt, i, sK, w_lo, mode, run ? ks.win_lo + (e_w - ks.n_sink) : -1, -1, lane, q0, q1,
      [&](int el) { return s_j[el]; },
      [&](int r, int el, int j, float dot) {
        float z = dot * sl2;
        if (a.alibi && j >= 0) {  // -m_h * min(i - j, L), in log2 units of the scaled logit
          const int dist = (a.L > 0) ? min(i - j, a.L) : (i - j);
          z -= exp2f(-8.f * (float)(g * REP + r + 1) / (float)a.Hq) * 1.4426950408889634f * (float)dist;
        }
        s_p[r][el] = (j >= 0) ? z : -CUDART_INF_F;
      });
  __syncthreads();
  // ---- per-head maximum, weights and their sum (warp r takes heads r, r + 4, ...) ----
  for (int r = warp; r < REP; r += NW) {
    float mx = -CUDART_INF_F;
    for (int e = lane; e < kChunk; e += 32) mx = fmaxf(mx, s_p[r][e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int e = lane; e < kChunk; e += 32) {
      const float p = (mx == -CUDART_INF_F) ? 0.f : ex2_approx(s_p[r][e] - mx);
      s_p[r][e] = p;
      sum += p;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
      s_m[r] = mx;
      s_l[r] = sum;
    }
  }
  if (!sw.wait(1, 2, kSiteDecodeV)) {
    sw.drain(2);
    return;
  }
  // ---- pass 2: O += p v (rows past the chunk's end are zeros with p = 0) ----
  float2 o0[REP][H], o1[REP][H];
#pragma unroll
  for (int r = 0; r < REP; ++r)
#pragma unroll
    for (int h = 0; h < H; ++h) o0[r][h] = o1[r][h] = make_float2(0.f, 0.f);
  for (int u0 = 0; u0 < KPW; u0 += KPS * UNR) {
    float2 v0[UNR][H], v1[UNR][H];
    int els[UNR];
#pragma unroll
    for (int x = 0; x < UNR; ++x) {
      els[x] = w_lo + u0 + x * KPS + kg;
      load_pairs<H>(sV + els[x] * D + p0, v0[x]);
      load_pairs<H>(sV + els[x] * D + p0 + half, v1[x]);
    }
#pragma unroll
    for (int x = 0; x < UNR; ++x) {
#pragma unroll
      for (int r = 0; r < REP; ++r) {
        const float p = s_p[r][els[x]];
        const float2 pp = make_float2(p, p);
#pragma unroll
        for (int h = 0; h < H; ++h) {
          o0[r][h] = ffma2(pp, v0[x][h], o0[r][h]);
          o1[r][h] = ffma2(pp, v1[x][h], o1[r][h]);
        }
      }
    }
  }
  // merge the warp's key slots (lanes sub, sub + LPK, ...), then the warps (fixed order)
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1)
#pragma unroll
    for (int r = 0; r < REP; ++r)
#pragma unroll
      for (int h = 0; h < H; ++h) {
        o0[r][h].x += __shfl_xor_sync(0xffffffffu, o0[r][h].x, o);
        o0[r][h].y += __shfl_xor_sync(0xffffffffu, o0[r][h].y, o);
        o1[r][h].x += __shfl_xor_sync(0xffffffffu, o1[r][h].x, o);
        o1[r][h].y += __shfl_xor_sync(0xffffffffu, o1[r][h].y, o);
      }
  if (kg == 0) {
#pragma unroll
    for (int r = 0; r < REP; ++r)
#pragma unroll
      for (int h = 0; h < H; ++h) {
        *reinterpret_cast<float2*>(&red_o[(warp * REP + r) * D + p0 + 2 * h]) = o0[r][h];
        *reinterpret_cast<float2*>(&red_o[(warp * REP + r) * D + p0 + 2 * h + half]) = o1[r][h];
      }
  }
  __syncthreads();
  for (int x = threadIdx.x; x < REP * D; x += kPartThreads) {
    const int r = x / D, c = x % D;
    float O = 0.f;
    for (int w = 0; w < NW; ++w) O += red_o[(w * REP + r) * D + c];
    const int h = g * REP + r;
    float* part = a.part + (((size_t)b * a.Hq + h) * a.n_chunks + blockIdx.y) * (D + 2);
    part[2 + c] = O;
    if (c == 0) {
      part[0] = s_m[r];
      part[1] = s_l[r];
    }
  }
}

// grid (B * Hq), kCombThreads threads: merge the chunk partials of one
// (batch, head), and the top-k keys' partial when there is one, into O and
// LSE.  Every load is issued before any arithmetic: the chunks' maxima and
// sums into shared memory, up to kCombRegs output partials per thread into
// registers (thread group q of G takes chunks q, q + G, ...); then the
// maximum, the weights 2^(m_x - M) and their sum, the weighted outputs, and
// the G groups added in a fixed order.
constexpr int kCombThreads = 512;
constexpr int kCombRegs = 8;
template <int D>
__global__ void __launch_bounds__(kCombThreads) decode_combine_kernel(DecodeArgs a) {
  constexpr int G = kCombThreads / D;
  constexpr int NWp = kCombThreads / 32;
  __shared__ float s_f[kMaxChunks + 1];  // chunk maxima, then weights
  __shared__ float s_s[kMaxChunks + 1];  // chunk sums
  __shared__ float s_red[G * D];
  __shared__ float s_ml[2];
  const int bh = blockIdx.x;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const KeySet ks = key_set(a, b);  // reads the block map, which preceded the split-K kernel
  const int nc0 = min((ks.n() + kChunk - 1) / kChunk, kMaxChunks);
  const int nc = nc0 + (a.tk_part ? 1 : 0);
  const float* part0 = a.part + (size_t)bh * a.n_chunks * (D + 2);
  auto slot = [&](int x) { return x < nc0 ? part0 + (size_t)x * (D + 2) : a.tk_part + (size_t)bh * (D + 2); };
  const int tid = threadIdx.x, q = tid / D, c = tid % D;
  grid_dep_wait();  // the partials
  float ov[kCombRegs];
#pragma unroll
  for (int u = 0; u < kCombRegs; ++u) {
    const int x = q + G * u;
    ov[u] = x < nc ? slot(x)[2 + c] : 0.f;
  }
  float mx = -CUDART_INF_F;
  for (int x = tid; x < nc; x += kCombThreads) {
    const float* sp = slot(x);
    const float m = sp[0];
    s_f[x] = m;
    s_s[x] = sp[1];
    mx = fmaxf(mx, m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) s_red[tid >> 5] = mx;
  __syncthreads();
  if (tid == 0) {
    float M = -CUDART_INF_F;
    for (int w = 0; w < NWp; ++w) M = fmaxf(M, s_red[w]);
    s_ml[0] = M;
  }
  __syncthreads();
  const float M = s_ml[0];
  float lsum = 0.f;
  for (int x = tid; x < nc; x += kCombThreads) {
    const float f = (s_f[x] == -CUDART_INF_F) ? 0.f : ex2_approx(s_f[x] - M);
    s_f[x] = f;
    lsum = fmaf(s_s[x], f, lsum);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  __syncthreads();  // s_red is reused
  if ((tid & 31) == 0) s_red[tid >> 5] = lsum;
  __syncthreads();
  if (tid == 0) {
    float L = 0.f;
    for (int w = 0; w < NWp; ++w) L += s_red[w];
    s_ml[1] = L;
  }
  float O = 0.f;
#pragma unroll
  for (int u = 0; u < kCombRegs; ++u) {
    const int x = q + G * u;
    if (x < nc) O = fmaf(s_f[x], ov[u], O);
  }
  for (int x = q + G * kCombRegs; x < nc; x += G) O = fmaf(s_f[x], slot(x)[2 + c], O);
  __syncthreads();  // s_red is reused
  s_red[q * D + c] = O;
  __syncthreads();
  if (q == 0) {
    float Ot = 0.f;
#pragma unroll
    for (int y = 0; y < G; ++y) Ot += s_red[y * D + c];
    const float L = s_ml[1];
    __nv_bfloat16* op = a.O + (size_t)b * a.o_sb + (size_t)h * a.o_sh;
    op[c] = __float2bfloat16_rn(L > 0.f ? Ot / L : 0.f);
    if (c == 0) a.lse[bh] = (L > 0.f) ? (M + __log2f(L)) * 0.69314718055994531f : -CUDART_INF_F;
  }
}

// ---------------------------------------------------------------------------
// top-k middle tokens of the decoding query ("LM-Infinite", section 方法,
// optional top-k): candidates n_start <= j < i - w that are not separators,
// ranked per query head by the unscaled logit (the capped one past L), ties
// to the smaller position.  Reading every candidate key is what the method
// asks for here; the K rows are read once per kv group.
// ---------------------------------------------------------------------------

// grid (B * Hkv, candidate chunks of kChunk positions): the chunk's K rows
// staged in shared memory, every candidate's logit for every query head of
// the group (the logit pass over consecutive positions), then per head the
// chunk's k best (separators excluded by their flag bit) into tk_cz / tk_cj:
// the top k of the whole row is the top k of the chunks' top k, so the
// selection merges k entries per chunk rather than every candidate.
template <int D, int REP>
__global__ void __launch_bounds__(kThreads) decode_topk_logits_kernel(DecodeArgs a) {
  using TL = Tiling<D, REP>;
  constexpr int EPL = TL::EPL, H = TL::H, LPK = TL::LPK, KPW = TL::KPW;
  extern __shared__ __align__(16) unsigned char dsm[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(dsm);  // [kChunk][D]
  __shared__ float s_z[REP][kChunk];
  __shared__ __align__(8) float s_qL[REP * D];  // R(L) q of the group's heads
  __shared__ RopeTab s_rt;
  __shared__ __align__(8) uint64_t s_bar[1];
  __shared__ int s_abort;
  grid_dep_launch();  // the selection kernel may be scheduled now; it waits for this grid
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x % a.Hkv, b = blockIdx.x / a.Hkv;
  const int i = a.T - 1;
  const int jend = i - a.window;  // candidates j < i - w
  const int j0 = a.n_start + blockIdx.y * kChunk;
  if (j0 >= jend) return;
  const __nv_bfloat16* kb = a.K + (size_t)b * a.k_sb + (size_t)g * a.k_sh;
  const int n_here = min(jend - j0, kChunk);
  // consecutive positions: one bulk copy when the rows are contiguous
  const bool bulk = a.k_st == D;
  if (threadIdx.x == 0) {
    s_abort = 0;
    if (bulk) {
      mbar_init(&s_bar[0], 1);
      fence_mbar_init();
    }
  }
  if (a.rope) load_rope_tab(a, s_rt, D / 2);
  __syncthreads();
  if (bulk) {
    if (threadIdx.x == 0) {
      const uint32_t bytes = (uint32_t)n_here * D * 2;
      mbar_expect_tx(&s_bar[0], bytes);
      bulk_copy(sK, kb + (size_t)j0 * D, bytes, &s_bar[0]);
    }
    zero_pieces(sK, n_here * D / 8, kChunk * D / 8, kThreads);
  } else {
    stage_rows<D, kThreads>(sK, kb, a.k_st, [&](int s) { return j0 + s < jend ? j0 + s : -1; });
    cp_async_commit();
  }
  StageWait sw{bulk, s_bar, &s_abort, a.status};
  // a warp whose candidates all lie past the cap scores the raw keys with
  // the query rotated to L; the others rotate their keys.  When the whole
  // chunk is past the cap, R(L) q is formed once per CTA in shared memory.
  constexpr int half = D / 2;
  const bool cta_capped = a.rope && a.L > 0 && i - (j0 + kChunk - 1) > a.L;
  if (cta_capped) {
    for (int x = threadIdx.x; x < REP * half; x += kThreads) {
      const int r = x / half, c = x % half;
      const float2 cs = rope_cs(s_rt, a.L, c);
      const __nv_bfloat16* qp = a.Q + (size_t)b * a.q_sb + (size_t)(g * REP + r) * a.q_sh;
      const float x0 = __bfloat162float(qp[c]), x1 = __bfloat162float(qp[c + half]);
      s_qL[r * D + c] = x0 * cs.x - x1 * cs.y;
      s_qL[r * D + c + half] = x1 * cs.x + x0 * cs.y;
    }
  }
  const int jw = j0 + warp * KPW;
  const bool all_capped = a.rope && a.L > 0 && i - (jw + KPW - 1) > a.L;
  const int mode = !a.rope || all_capped ? kRotNone : kRotRun;
  const int p0 = (lane % LPK) * EPL;
  float2 q0[REP][H], q1[REP][H];
  if (!cta_capped) load_query<D, REP>(a, b, g, p0, q0, q1);
  const uint2* words = a.sep_words ? a.sep_words + (size_t)b * (a.T / 32 + 1) : nullptr;
  if (!sw.wait(0, 1, kSiteTopkK)) {
    sw.drain(1);
    return;
  }
  if (cta_capped) {
#pragma unroll
    for (int r = 0; r < REP; ++r)
#pragma unroll
      for (int h = 0; h < H; ++h) {
        q0[r][h] = *reinterpret_cast<const float2*>(&s_qL[r * D + p0 + 2 * h]);
        q1[r][h] = *reinterpret_cast<const float2*>(&s_qL[r * D + p0 + 2 * h + half]);
      }
  }
  logits_pass<D, REP, kThreads / 32>(
      a, s_rt, i, sK, warp * KPW, mode, jw, all_capped && !cta_capped ? a.L : -1, lane, q0, q1,
      [&](int el) { return j0 + el < jend ? j0 + el : -1; },
      [&](int r, int el, int j, float dot) {
        const bool sep = j >= 0 && words && ((__ldg(&words[j >> 5].y) >> (j & 31)) & 1u);
        s_z[r][el] = (j >= 0 && !sep) ? dot : -CUDART_INF_F;
      });
  __syncthreads();
  // per head: k rounds of a warp argmax by (z desc, j asc) over the chunk
  // (lane l holds keys l, l + 32, l + 64, l + 96)
  const int k = a.topk;
  const int chunk = blockIdx.y;
  for (int r = warp; r < REP; r += kThreads / 32) {
    float zv[kChunk / 32];
    int jv[kChunk / 32];
#pragma unroll
    for (int u = 0; u < kChunk / 32; ++u) {
      const int el = lane + 32 * u;
      zv[u] = s_z[r][el];
      jv[u] = (zv[u] == -CUDART_INF_F) ? -1 : j0 + el;
    }
    const size_t base = (((size_t)b * a.Hq + (size_t)g * REP + r) * a.tk_nchunks + chunk) * k;
    for (int y = 0; y < k; ++y) {
      float bz = -CUDART_INF_F;
      int bj = -1;
#pragma unroll
      for (int u = 0; u < kChunk / 32; ++u)
        if (sel_before(zv[u], jv[u], bz, bj)) {
          bz = zv[u];
          bj = jv[u];
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        if (sel_before(oz, oj, bz, bj)) {
          bz = oz;
          bj = oj;
        }
      }
#pragma unroll
      for (int u = 0; u < kChunk / 32; ++u)
        if (jv[u] == bj && bj >= 0) {  // the winner leaves its list (positions are distinct)
          jv[u] = -1;
          zv[u] = -CUDART_INF_F;
        }
      if (lane == 0) {
        a.tk_cz[base + y] = bj >= 0 ? bz : -CUDART_INF_F;
        a.tk_cj[base + y] = bj;
      }
    }
  }
}


constexpr int kSelThreads = 512;
constexpr int kSelMaxK = 16;

// grid (B * Hq): the k best candidates of one (batch, head) from the chunks'
// top k -- a strided pass keeping a sorted list per thread, then k rounds of
// a block argmax -- written out, and the selected keys' softmax partial
// (their maximum, sum of weights and weighted V rows) for the chunk merge.
template <int D>
__global__ void __launch_bounds__(kSelThreads) decode_topk_select_kernel(DecodeArgs a) {
  __shared__ float red_z[kSelThreads / 32];
  __shared__ int red_j[kSelThreads / 32];
  __shared__ float s_z[kSelMaxK];
  __shared__ int s_j[kSelMaxK];
  grid_dep_launch();  // the split-K kernel may start its K / V copies now
  const int bh = blockIdx.x;
  const int b = bh / a.Hq, h = bh % a.Hq, g = h / (a.Hq / a.Hkv);
  grid_dep_wait();  // the chunks' picks
  const int n_c = a.tk_nchunks * a.topk;  // the chunks' picks (-1 padding)
  const float* czr = a.tk_cz + (size_t)bh * n_c;
  const int32_t* cjr = a.tk_cj + (size_t)bh * n_c;
  float vals[kSelMaxK];
  int idxs[kSelMaxK];
#pragma unroll
  for (int y = 0; y < kSelMaxK; ++y) {
    vals[y] = -CUDART_INF_F;
    idxs[y] = -1;
  }
  // each thread visits its entries in increasing position order (chunks in
  // order, each chunk's picks by (z desc, j asc) but a thread sees one
  // chunk's entries a stride apart), so ties are settled by position
  for (int e = (int)threadIdx.x; e < n_c; e += kSelThreads) {
    const int j = cjr[e];
    if (j < 0) continue;
    const float z = czr[e];
    if (sel_before(z, j, vals[kSelMaxK - 1], idxs[kSelMaxK - 1])) {
      float v = z;
      int jj = j;
#pragma unroll
      for (int y = 0; y < kSelMaxK; ++y) {
        if (sel_before(v, jj, vals[y], idxs[y])) {
          const float tv = vals[y];
          const int tj = idxs[y];
          vals[y] = v;
          idxs[y] = jj;
          v = tv;
          jj = tj;
        }
      }
    }
  }
  block_topk_rounds<kSelMaxK>(a.topk, vals, idxs, red_z, red_j, [&](int r, float wz, int wj) {
    s_j[r] = wj;
    s_z[r] = wj >= 0 ? wz : -CUDART_INF_F;
  });
  __syncthreads();
  const int k = a.topk;
  if ((int)threadIdx.x < k) {
    a.tk_idx[(size_t)bh * k + threadIdx.x] = s_j[threadIdx.x];
    a.tk_z[(size_t)bh * k + threadIdx.x] = s_z[threadIdx.x];
  }
  // scaled log2-unit logits of the picks; with ALiBi every candidate is
  // past the cap (w >= L) and takes -m_h L
  const float sl2 = a.scale_log2;
  const float bias = a.alibi ? exp2f(-8.f * (float)(h + 1) / (float)a.Hq) * 1.4426950408889634f * (float)a.L : 0.f;
  float m = -CUDART_INF_F;
  for (int r = 0; r < k; ++r)
    if (s_j[r] >= 0) m = fmaxf(m, s_z[r] * sl2 - bias);
  float* part = a.tk_part + (size_t)bh * (D + 2);
  const __nv_bfloat16* vb = a.V + (size_t)b * a.v_sb + (size_t)g * a.v_sh;
  for (int c = threadIdx.x; c < D; c += kSelThreads) {
    float l = 0.f, o = 0.f;
    for (int r = 0; r < k; ++r) {
      if (s_j[r] < 0) continue;
      const float p = ex2_approx(s_z[r] * sl2 - bias - m);
      l += p;
      o = fmaf(p, __bfloat162float(vb[(size_t)s_j[r] * a.v_st + c]), o);
    }
    part[2 + c] = o;
    if (c == 0) {
      part[0] = m;
      part[1] = l;
    }
  }
}

template <class Kern>
cudaError_t launch_k(Kern kern, dim3 grid, int threads, size_t smem, bool pdl, const DecodeArgs& a,
                     cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

// dynamic shared memory above the default 48 KB
template <class Kern>
cudaError_t allow_smem(Kern kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int D, int REP>
cudaError_t launch_dr(const DecodeArgs& a0, cudaStream_t st) {
  // the rotation by KPS positions that steps a lane from one of its keys to
  // the next along a run, from the angle in double
  DecodeArgs a = a0;
  constexpr int KPS = Tiling<D, REP>::KPS;
  for (int c = 0; c < D / 2; ++c) {
    const double ang = KPS * a.rope_scale * a.inv_freq[c];
    a.step_cs[c] = a.rope ? make_float2((float)std::cos(ang), (float)std::sin(ang)) : make_float2(1.f, 0.f);
    // turns per position as a sum of two floats
    const double f = a.rope_scale * a.inv_freq[c] / 6.283185307179586;
    a.turn_hi[c] = (float)f;
    a.turn_lo[c] = (float)(f - (double)a.turn_hi[c]);
  }
  // without separators or per-sequence lengths the kept-key count is a
  // closed form: launch exactly its chunks
  int chunks = a.n_chunks;
  if (!a.sep_words && !a.seq_len) {
    const int i = a.T - 1, ns = std::min(a.n_start, a.T);
    const int win_lo = std::max(ns, i - a.window);
    chunks = std::min(chunks, std::max(1, (ns + std::max(0, i - win_lo + 1) + kChunk - 1) / kChunk));
  }
  const size_t rows_bytes = (size_t)kChunk * D * sizeof(__nv_bfloat16);
  cudaError_t e;
  bool after_kernel = false;  // a kernel of this step precedes the next launch in the stream
  if (a.topk > 0) {
    const int ncand = a.T - 1 - a.window - a.n_start;
    if (ncand > 0) {
      e = allow_smem(decode_topk_logits_kernel<D, REP>, rows_bytes);
      if (e != cudaSuccess) return e;
      e = launch_k(decode_topk_logits_kernel<D, REP>, dim3(a.B * a.Hkv, a.tk_nchunks), kThreads, rows_bytes, false,
                   a, st);
      if (e != cudaSuccess) return e;
      after_kernel = true;
    }
    e = launch_k(decode_topk_select_kernel<D>, dim3(a.B * a.Hq), kSelThreads, 0, after_kernel, a, st);
    if (e != cudaSuccess) return e;
    after_kernel = true;
  }
  e = allow_smem(decode_partial_kernel<D, REP>, 2 * rows_bytes);
  if (e != cudaSuccess) return e;
  e = launch_k(decode_partial_kernel<D, REP>, dim3(a.B * a.Hkv, chunks), PartCfg<REP>::NT, 2 * rows_bytes,
               after_kernel, a, st);
  if (e != cudaSuccess) return e;
  return launch_k(decode_combine_kernel<D>, dim3(a.B * a.Hq), kCombThreads, 0, true, a, st);
}

template <int D>
cudaError_t launch_d(const DecodeArgs& a, cudaStream_t st) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_dr<D, 1>(a, st);
    case 2: return launch_dr<D, 2>(a, st);
    case 4: return launch_dr<D, 4>(a, st);
    case 8: return launch_dr<D, 8>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int decode_chunks(int T) { return (T + kChunk - 1) / kChunk; }
int decode_topk_chunks(int n_candidates) { return n_candidates > 0 ? (n_candidates + kChunk - 1) / kChunk : 0; }
int decode_max_len() { return kMaxChunks * kChunk; }

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  if (a.d / 2 > (int)(sizeof(a.inv_freq) / sizeof(a.inv_freq[0]))) return cudaErrorInvalidValue;
  if (a.d == 128) return launch_d<128>(a, st);
  if (a.d == 64) return launch_d<64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace sattn
