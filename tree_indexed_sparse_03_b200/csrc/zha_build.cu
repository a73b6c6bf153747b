// Tree build and append kernels.
//
// Method ("Zyphra Hierarchical Attention", Zyphra blog, section "Building the
// tree"; tanhow.com summary, section "How does ZHA's tree indexer work? /
// Building the tree"): contiguous blocks of `block` raw keys are summarised at
// each reference query r_j by the tangent plane of their log attention mass
// f_B(r_j) = log sum_k exp(r_j.k/sqrt(d)): value f, slope mu_j/sqrt(d) with
// mu_j the softmax-weighted mean key, intercept b_j = f - r_j.mu_j/sqrt(d).
// Summaries are merged exactly, `block` children per parent: parent f is the
// logsumexp of the children's f, parent mu_j the children's mu_j weighted by
// the softmax of their f(r_j).
//
// GPU arithmetic (fp32, fixed order, identical for build and append):
//   leaf:  s_k = (r_j . k) * (1/sqrt d)      (sequential fma over d)
//          m = max s, Z = sum exp(s - m), f = m + log Z, w_k = exp(s_k - m) / Z
//          g = sum_k w_k s_k  (= r_j.mu_j/sqrt d exactly),  mu_j = sum_k w_k k
//   merge: m = max f_c, Z = sum exp(f_c - m), f = m + log Z, a_c = exp(f_c - m) / Z
//          g = sum_c a_c g_c,  mu_j = sum_c a_c mu_c
//   store: mu rounded to the element type, b_j = f - g and f in fp32.
// Every merge reads its children's unrounded fp32 values.  Levels 1..S (S =
// chunk level, b^S <= 64 keys, or S = 1 when b > 64) are computed inside one
// CTA per aligned chunk of b^S keys; the chunk roots (level S) and the levels
// above are kept in fp32 as well, and levels S+1..L are merged from them by
// upper_kernel.  An append recomputes the chunks that gain complete leaves
// and writes only the nodes that became complete, so build(n) followed by
// append(m) stores exactly the same bits as build(n + m); an append that
// completes no node of levels 2..S (most single tokens) computes only its new
// leaves, in one kernel that also copies the rows.
#include <type_traits>

#include "zha_args.cuh"

namespace zha {

constexpr int kBuildThreads = 256;

struct ChunkSmem {
  int CK, KS, RG, NN;
  size_t keys, refs, refb, w, wa, mu, fs, gs, total;
};

template <typename T, int D>
__host__ __device__ inline ChunkSmem chunk_smem_layout(int block, int chunk_level, int R) {
  ChunkSmem L;
  int CK = 1;
  for (int i = 0; i < chunk_level; ++i) CK *= block;
  L.CK = CK;
  L.KS = D + 16 / int(sizeof(T));  // key row stride in elements (16-byte pad)
  L.RG = R < 4 ? R : 4;
  int nn = 0, w = CK, na = 0;
  for (int l = 1; l <= chunk_level; ++l) {
    w /= block;
    nn += w;
    if (l >= 2) na += w * block;  // children of the level-l nodes
  }
  L.NN = nn;
  size_t off = 0;
  L.keys = off; off += size_t(CK) * L.KS * sizeof(T); off = (off + 15) & ~size_t(15);
  L.refs = off; off += size_t(R) * (D + 1) * 4;                     // fp32 refs (scalar scores)
  off = (off + 15) & ~size_t(15);
  L.refb = off; off += size_t(R) * D * 2;                           // bf16 refs (tensor-core scores)
  L.w = off;    off += size_t(CK) * R * 4;                          // leaf scores, then softmax weights
  L.wa = off;   off += size_t(na > 0 ? na : 1) * R * 4;             // merge weights of the children
  off = (off + 15) & ~size_t(15);
  L.mu = off;   off += size_t(nn) * L.RG * D * 4;                   // fp32 slopes of one group of refs
  L.fs = off;   off += size_t(nn) * R * 4;
  L.gs = off;   off += size_t(nn) * R * 4;
  L.total = (off + 15) & ~size_t(15);
  return L;
}

// Scores s[k][j] = (r_j . key_k) / sqrt(d) of nkeys keys (rows of `keys`, stride KS elements) and R bf16
// reference rows (`refb`, [R][D]) on the tensor cores: mma.sync m16n8k16, 16 keys x 8 refs per tile, the D
// dimensions in 16-wide steps accumulated in order from zero.  Each score depends only on its key, its
// reference query and this fixed sequence, so every caller (build, append) gets the same bits.  Warps take
// tiles in turn; scores go to sc[k * R + j].
template <int D>
__device__ __forceinline__ void scores_mma(const __nv_bfloat16* keys, int KS, int nkeys,
                                           const __nv_bfloat16* refb, int R, float inv_sqrt_d, float* sc,
                                           int warp, int nwarps) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
  const int mt = (nkeys + 15) / 16, nt = (R + 7) / 8;
  for (int tile = warp; tile < mt * nt; tile += nwarps) {
    const int m0 = (tile / nt) * 16, n0 = (tile % nt) * 8;
    const int r0 = min(m0 + g, nkeys - 1), r1 = min(m0 + g + 8, nkeys - 1);  // rows past nkeys: masked
    const int c = min(n0 + g, R - 1);
    const __nv_bfloat16* a0p = keys + size_t(r0) * KS + 2 * t4;
    const __nv_bfloat16* a1p = keys + size_t(r1) * KS + 2 * t4;
    const __nv_bfloat16* bp = refb + size_t(c) * D + 2 * t4;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k0 = 0; k0 < D; k0 += 16) {
      const uint32_t a[4] = {*reinterpret_cast<const uint32_t*>(a0p + k0), *reinterpret_cast<const uint32_t*>(a1p + k0),
                             *reinterpret_cast<const uint32_t*>(a0p + k0 + 8),
                             *reinterpret_cast<const uint32_t*>(a1p + k0 + 8)};
      const uint32_t bb[2] = {*reinterpret_cast<const uint32_t*>(bp + k0), *reinterpret_cast<const uint32_t*>(bp + k0 + 8)};
      mma_bf16_16816(acc, a, bb);
    }
    const int row0 = m0 + g, row1 = m0 + g + 8, col = n0 + 2 * t4;
    if (row0 < nkeys) {
      if (col < R) sc[row0 * R + col] = __fmul_rn(acc[0], inv_sqrt_d);
      if (col + 1 < R) sc[row0 * R + col + 1] = __fmul_rn(acc[1], inv_sqrt_d);
    }
    if (row1 < nkeys) {
      if (col < R) sc[row1 * R + col] = __fmul_rn(acc[2], inv_sqrt_d);
      if (col + 1 < R) sc[row1 * R + col + 1] = __fmul_rn(acc[3], inv_sqrt_d);
    }
  }
}

// Scores of the fp32 configurations: sequential fma over the dimensions.
template <typename T, int D>
__device__ __forceinline__ void scores_fma(const T* keys, int KS, int nkeys, const float* refs, int R,
                                           float inv_sqrt_d, float* sc) {
  using E = Elem<T>;
  for (int i = threadIdx.x; i < nkeys * R; i += blockDim.x) {
    const int k = i / R, j = i - (i / R) * R;
    const T* kr = keys + size_t(k) * KS;
    const float* rr = refs + j * (D + 1);
    float acc = 0.f;
#pragma unroll 8
    for (int e = 0; e < D; ++e) acc = __fmaf_rn(E::to_f(kr[e]), rr[e], acc);
    sc[k * R + j] = __fmul_rn(acc, inv_sqrt_d);
  }
}

// Leaf value, projected mean score and softmax weights of (leaf li, ref j): m = max s, Z = sum exp(s - m),
// f = m + log Z, w_k = exp(s_k - m) / Z (written over the scores), g = sum_k w_k s_k.
__device__ __forceinline__ void leaf_softmax(float* s, int stride, int b, float* f_out, float* g_out) {
  float m = -INFINITY;
  for (int k = 0; k < b; ++k) m = fmaxf(m, s[k * stride]);
  float Z = 0.f;
  for (int k = 0; k < b; ++k) Z = __fadd_rn(Z, expf(__fsub_rn(s[k * stride], m)));
  const float f = __fadd_rn(m, logf(Z));
  float g = 0.f;
  for (int k = 0; k < b; ++k) {
    const float wk = __fdiv_rn(expf(__fsub_rn(s[k * stride], m)), Z);
    g = __fmaf_rn(wk, s[k * stride], g);
    s[k * stride] = wk;
  }
  *f_out = f;
  *g_out = g;
}

// Eight consecutive values of a row (fp32) -> the element type, stored as one or two 16-byte vectors.
template <typename T>
__device__ __forceinline__ void store8(T* dst, const float (&v)[8]);
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* dst, const float (&v)[8]) {
  uint4 o;
  o.x = pack_bf16(v[0], v[1]);
  o.y = pack_bf16(v[2], v[3]);
  o.z = pack_bf16(v[4], v[5]);
  o.w = pack_bf16(v[6], v[7]);
  *reinterpret_cast<uint4*>(dst) = o;
}
template <>
__device__ __forceinline__ void store8<float>(float* dst, const float (&v)[8]) {
  *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8f(float* dst, const float (&v)[8]) {
  *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// One CTA per (chunk, KV head).  Computes every complete node of levels
// 1..S inside the chunk and writes those with index >= the previous count.
// Scores of all keys and reference queries first (tensor cores for bf16),
// then the softmax weights of the leaves and of every merge (all reference
// queries), then per group of RG reference queries the fp32 slopes, level by
// level, each thread producing eight consecutive dimensions of a row (the
// same arithmetic per value: children in order), written to the records as
// 16-byte vectors.
template <typename T, int D>
__global__ void __launch_bounds__(kBuildThreads) chunk_kernel(TreeDev t, int64_t n_tokens,
                                                              int64_t n_old, int64_t chunk0) {
  using E = Elem<T>;
  constexpr bool kMma = std::is_same<T, __nv_bfloat16>::value;
  const int h = blockIdx.y;
  const int64_t chunk = chunk0 + blockIdx.x;
  const int b = t.block, S = t.chunk_level, R = t.refs;
  const ChunkSmem L = chunk_smem_layout<T, D>(b, S, R);
  const int CK = L.CK, KS = L.KS, RG = L.RG;
  const int64_t n1 = n_tokens / b;
  const int64_t leaves_per_chunk = CK / b;
  const int64_t leaf0 = chunk * leaves_per_chunk;
  const int nleaves = int(min64(leaves_per_chunk, n1 - leaf0));
  if (nleaves <= 0) return;
  const int nkeys = nleaves * b;
  const int64_t key0 = chunk * CK;
  const int tid = threadIdx.x, warp = tid >> 5;

  extern __shared__ __align__(16) unsigned char smem[];
  T* keys = reinterpret_cast<T*>(smem + L.keys);
  float* refs = reinterpret_cast<float*>(smem + L.refs);
  __nv_bfloat16* refb = reinterpret_cast<__nv_bfloat16*>(smem + L.refb);
  float* w = reinterpret_cast<float*>(smem + L.w);
  float* wa = reinterpret_cast<float*>(smem + L.wa);
  float* mu = reinterpret_cast<float*>(smem + L.mu);
  float* fs = reinterpret_cast<float*>(smem + L.fs);
  float* gs = reinterpret_cast<float*>(smem + L.gs);

  // Stage the chunk's complete keys (16-byte vectors) and the refs.
  {
    constexpr int VPR = D * sizeof(T) / 16;  // vectors per key row
    const T* Kh = static_cast<const T*>(t.K) + (size_t(h) * t.capacity + key0) * D;
    for (int i = tid; i < nkeys * VPR; i += blockDim.x) {
      const int k = i / VPR, v = i % VPR;
      uint4 x = ldg_stream(Kh + size_t(k) * D + v * (16 / sizeof(T)));
      *reinterpret_cast<uint4*>(keys + size_t(k) * KS + v * (16 / sizeof(T))) = x;
    }
    const T* Rh = static_cast<const T*>(t.refsp) + size_t(h) * R * D;
    if constexpr (kMma) {
      for (int i = tid; i < R * D; i += blockDim.x) refb[i] = Rh[i];
    } else {
      for (int i = tid; i < R * D; i += blockDim.x) refs[(i / D) * (D + 1) + i % D] = E::to_f(Rh[i]);
    }
  }
  __syncthreads();

  // node slot of (level, index-in-chunk) inside the per-chunk arrays, and the first merge weight of each level
  int slot_off[kMaxLevels + 1], wa_off[kMaxLevels + 1];
  {
    int off = 0, aoff = 0, wdt = CK;
    for (int l = 1; l <= S; ++l) {
      slot_off[l] = off;
      wa_off[l] = aoff;
      wdt /= b;
      off += wdt;
      if (l >= 2) aoff += wdt * b;
    }
  }
  auto slot = [&](int level, int i) { return slot_off[level] + i; };
  auto nval_of = [&](int level) {
    const int64_t pw = t.pow_b[level], per_chunk = CK / pw;
    return int(min64(per_chunk, n_tokens / pw - chunk * per_chunk));
  };

  // scores of every key and reference query
  if constexpr (kMma) scores_mma<D>(keys, KS, nkeys, refb, R, t.inv_sqrt_d, w, warp, kBuildThreads / 32);
  else scores_fma<T, D>(keys, KS, nkeys, refs, R, t.inv_sqrt_d, w);
  __syncthreads();
  // leaf values and weights, all reference queries
  for (int i = tid; i < nleaves * R; i += blockDim.x) {
    const int li = i / R, j = i - li * R;
    leaf_softmax(w + (li * b) * R + j, R, b, &fs[slot(1, li) * R + j], &gs[slot(1, li) * R + j]);
  }
  __syncthreads();
  // merge values and weights of levels 2..S, all reference queries
  for (int level = 2; level <= S; ++level) {
    const int nval = nval_of(level);
    for (int i = tid; i < nval * R; i += blockDim.x) {
      const int ni = i / R, j = i - ni * R;
      const int c0 = slot(level - 1, ni * b);
      float m = -INFINITY;
      for (int c = 0; c < b; ++c) m = fmaxf(m, fs[(c0 + c) * R + j]);
      float Z = 0.f;
      for (int c = 0; c < b; ++c) Z = __fadd_rn(Z, expf(__fsub_rn(fs[(c0 + c) * R + j], m)));
      const float f = __fadd_rn(m, logf(Z));
      float g = 0.f;
      for (int c = 0; c < b; ++c) {
        const float a = __fdiv_rn(expf(__fsub_rn(fs[(c0 + c) * R + j], m)), Z);
        wa[(wa_off[level] + ni * b + c) * R + j] = a;
        g = __fmaf_rn(a, gs[(c0 + c) * R + j], g);
      }
      fs[slot(level, ni) * R + j] = f;
      gs[slot(level, ni) * R + j] = g;
    }
    __syncthreads();
  }

  // slopes: rows (node, ref of the group) of D values, 8 consecutive values per thread
  constexpr int VEC = 8, TPR = D / VEC, RPI = kBuildThreads / TPR;
  const int e0 = (tid % TPR) * VEC;
  for (int j0 = 0; j0 < R; j0 += RG) {
    const int rg = min(RG, R - j0);
    for (int level = 1; level <= S; ++level) {
      const int64_t pw = t.pow_b[level];
      const int64_t base = chunk * (CK / pw);
      const int nval = nval_of(level);
      const int64_t first_new = n_old / pw;
      const bool keep32 = (level == S) && (S < t.levels);
      for (int row = tid / TPR; row < nval * rg; row += RPI) {
        const int ni = row / rg, jj = row - ni * rg, j = j0 + jj;
        float acc[VEC];
#pragma unroll
        for (int q = 0; q < VEC; ++q) acc[q] = 0.f;
        if (level == 1) {
          for (int k = 0; k < b; ++k) {
            const float wk = w[(ni * b + k) * R + j];
            float x[VEC];
            if constexpr (sizeof(T) == 2) {
              unpack16<T>(*reinterpret_cast<const uint4*>(keys + size_t(ni * b + k) * KS + e0), x);
            } else {
              unpack16<T>(*reinterpret_cast<const uint4*>(keys + size_t(ni * b + k) * KS + e0), x);
              unpack16<T>(*reinterpret_cast<const uint4*>(keys + size_t(ni * b + k) * KS + e0 + 4), x + 4);
            }
#pragma unroll
            for (int q = 0; q < VEC; ++q) acc[q] = __fmaf_rn(wk, x[q], acc[q]);
          }
        } else {
          const int c0 = slot(level - 1, ni * b);
          for (int c = 0; c < b; ++c) {
            const float a = wa[(wa_off[level] + ni * b + c) * R + j];
            const float* src = mu + (size_t(c0 + c) * RG + jj) * D + e0;
            const float4 u0 = *reinterpret_cast<const float4*>(src), u1 = *reinterpret_cast<const float4*>(src + 4);
            const float x[VEC] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int q = 0; q < VEC; ++q) acc[q] = __fmaf_rn(a, x[q], acc[q]);
          }
        }
        store8f(mu + (size_t(slot(level, ni)) * RG + jj) * D + e0, acc);
        const int64_t gi = base + ni;
        if (gi >= first_new) {
          store8<T>(reinterpret_cast<T*>(t.rec(level, h, gi)) + size_t(j) * D + e0, acc);
          if (keep32) store8f(t.up(level, h, gi) + size_t(j) * D + e0, acc);
        }
      }
      __syncthreads();
    }
  }
  // intercepts and values of the nodes that are new in this call (and their fp32 copies at the chunk level),
  // the padding after bias[R] zeroed
  const int padded = int((t.rec_bytes - size_t(R) * D * sizeof(T)) / 4);
  for (int level = 1; level <= S; ++level) {
    const int64_t pw = t.pow_b[level];
    const int64_t base = chunk * (CK / pw);
    const int nval = nval_of(level);
    const int64_t first_new = n_old / pw;
    const bool keep32 = (level == S) && (S < t.levels);
    for (int i = tid; i < nval * padded; i += blockDim.x) {
      const int ni = i / padded, j = i - ni * padded;
      const int64_t gi = base + ni;
      if (gi < first_new) continue;
      float* bias = reinterpret_cast<float*>(t.rec(level, h, gi) + size_t(R) * D * sizeof(T));
      if (j >= R) {
        bias[j] = 0.f;
        continue;
      }
      const float f = fs[slot(level, ni) * R + j];
      const float g = gs[slot(level, ni) * R + j];
      bias[j] = __fsub_rn(f, g);
      t.fval(level, h, gi)[j] = f;
      if (keep32) {
        float* u = t.up(level, h, gi);
        u[size_t(R) * D + j] = f;
        u[size_t(R) * D + R + j] = g;
      }
    }
  }
}

// One CTA per (new node, KV head) at a level above the chunk level.
template <typename T, int D>
__global__ void __launch_bounds__(kBuildThreads) upper_kernel(TreeDev t, int level, int64_t first) {
  using E = Elem<T>;
  const int h = blockIdx.y;
  const int64_t gi = first + blockIdx.x;
  const int b = t.block, R = t.refs;
  extern __shared__ __align__(16) unsigned char smem[];
  float* a = reinterpret_cast<float*>(smem);  // [b][R]
  float* fg = a + size_t(b) * R;               // f[R], g[R]
  const int tid = threadIdx.x;
  for (int j = tid; j < R; j += blockDim.x) {
    float m = -INFINITY;
    for (int c = 0; c < b; ++c) m = fmaxf(m, t.up(level - 1, h, gi * b + c)[size_t(R) * D + j]);
    float Z = 0.f;
    for (int c = 0; c < b; ++c)
      Z = __fadd_rn(Z, expf(__fsub_rn(t.up(level - 1, h, gi * b + c)[size_t(R) * D + j], m)));
    const float f = __fadd_rn(m, logf(Z));
    float g = 0.f;
    for (int c = 0; c < b; ++c) {
      const float* u = t.up(level - 1, h, gi * b + c);
      const float ac = __fdiv_rn(expf(__fsub_rn(u[size_t(R) * D + j], m)), Z);
      a[c * R + j] = ac;
      g = __fmaf_rn(ac, u[size_t(R) * D + R + j], g);
    }
    fg[j] = f;
    fg[R + j] = g;
  }
  __syncthreads();
  const bool keep32 = level < t.levels;
  T* rec = reinterpret_cast<T*>(t.rec(level, h, gi));
  for (int i = tid; i < R * D; i += blockDim.x) {
    const int j = i / D;
    float acc = 0.f;
    for (int c = 0; c < b; ++c) acc = __fmaf_rn(a[c * R + j], t.up(level - 1, h, gi * b + c)[i], acc);
    rec[i] = E::from_f(acc);
    if (keep32) t.up(level, h, gi)[i] = acc;
  }
  float* bias = reinterpret_cast<float*>(t.rec(level, h, gi) + size_t(R) * D * sizeof(T));
  const int padded = int((t.rec_bytes - size_t(R) * D * sizeof(T)) / 4);
  for (int j = tid; j < padded; j += blockDim.x) bias[j] = j < R ? __fsub_rn(fg[j], fg[R + j]) : 0.f;
  for (int j = tid; j < R; j += blockDim.x) {
    t.fval(level, h, gi)[j] = fg[j];
    if (keep32) {
      float* u = t.up(level, h, gi);
      u[size_t(R) * D + j] = fg[j];
      u[size_t(R) * D + R + j] = fg[R + j];
    }
  }
}

// FP4 router records of the nodes [first, first + gridDim.x) of one level, from
// the stored records: one thread per (reference row, group of 16 dimensions)
// quantises the group (scale = e4m3(amax / 6), codes = e2m1(v / scale), both
// rounded to nearest, ties to even) and writes its 8 code bytes and its scale
// byte; the intercepts are copied and the padding zeroed.
template <typename T, int D>
__global__ void quant4_kernel(TreeDev t, int level, int64_t first) {
  using E = Elem<T>;
  const int h = blockIdx.y;
  const int64_t gi = first + blockIdx.x;
  const int R = t.refs;
  constexpr int G = D / 16;
  const T* src = reinterpret_cast<const T*>(t.rec(level, h, gi));
  unsigned char* dst = reinterpret_cast<unsigned char*>(t.rec4(level, h, gi));
  for (int i = threadIdx.x; i < R * G; i += blockDim.x) {
    const int j = i / G, g = i % G;
    float v[16];
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      v[k] = E::to_f(src[size_t(j) * D + g * 16 + k]);
      amax = fmaxf(amax, fabsf(v[k]));
    }
    uint32_t sbits;
    const float sc = e4m3_nearest(__fdiv_rn(amax, 6.f), &sbits);
    uint32_t w0 = 0u, w1 = 0u;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t c = sc > 0.f ? e2m1_code(__fdiv_rn(v[k], sc)) : 0u;
      if (k < 8) w0 |= c << (4 * k);
      else w1 |= c << (4 * (k - 8));
    }
    *reinterpret_cast<uint2*>(dst + size_t(j) * (D / 2) + g * 8) = make_uint2(w0, w1);
    dst[size_t(R) * (D / 2) + size_t(j) * G + g] = (unsigned char)sbits;
  }
  const float* bsrc = reinterpret_cast<const float*>(t.rec(level, h, gi) + size_t(R) * D * sizeof(T));
  float* bdst = reinterpret_cast<float*>(dst + size_t(R) * (D / 2 + G));
  const int padded = int((t.rec4_bytes - size_t(R) * (D / 2 + G)) / 4);
  for (int j = threadIdx.x; j < padded; j += blockDim.x) bdst[j] = j < R ? bsrc[j] : 0.f;
}


// Appends that complete no node of levels 2..S (most single tokens): one CTA
// per KV head copies the new rows and computes only the newly completed leaves,
// with the chunk kernel's arithmetic in the same order (sequential fma over the
// dimensions for each score, the leaf's softmax over its keys in key order),
// so the stored bits equal those of a full build.  Levels above the chunk
// level are merged afterwards by upper_kernel as usual.
constexpr int kAppendThreads = 256;
constexpr int kAppendMaxBlock = 64;  // keys per leaf the fast path stages

template <typename T, int D>
__global__ void __launch_bounds__(kAppendThreads) append_fast_kernel(TreeDev t, const T* Knew, const T* Vnew,
                                                                     int64_t n_old, int64_t m) {
  using E = Elem<T>;
  constexpr bool kMma = std::is_same<T, __nv_bfloat16>::value;
  constexpr int VPR = D * sizeof(T) / 16;
  const int h = blockIdx.x, tid = threadIdx.x;
  const int b = t.block, R = t.refs;
  extern __shared__ __align__(16) unsigned char smem[];
  T* keys = reinterpret_cast<T*>(smem);                                              // [b][D]
  float* refs = reinterpret_cast<float*>(smem + size_t(kAppendMaxBlock) * D * sizeof(T));  // [R][D + 1]
  __nv_bfloat16* refb = reinterpret_cast<__nv_bfloat16*>(refs + size_t(kMaxRefs) * (D + 1));  // [R][D]
  float* sc = reinterpret_cast<float*>(refb + size_t(kMaxRefs) * D);                 // [b][R]
  float* fg = sc + size_t(kAppendMaxBlock) * kMaxRefs;                                // [R] f, [R] g
  // the new rows of this head (rows are [Hkv][m][d]: head h's rows are contiguous)
  for (int64_t i = tid; i < m * VPR; i += blockDim.x) {
    const int64_t r = i / VPR, v = i % VPR;
    const size_t src = (size_t(h) * m + r) * D + v * (16 / sizeof(T));
    const size_t dst = (size_t(h) * t.capacity + n_old + r) * D + v * (16 / sizeof(T));
    *reinterpret_cast<uint4*>(static_cast<T*>(t.K) + dst) = *reinterpret_cast<const uint4*>(Knew + src);
    *reinterpret_cast<uint4*>(static_cast<T*>(t.V) + dst) = *reinterpret_cast<const uint4*>(Vnew + src);
  }
  const int64_t l0 = n_old / b, l1 = (n_old + m) / b;
  if (l1 == l0) return;
  const T* Rh = static_cast<const T*>(t.refsp) + size_t(h) * R * D;
  if constexpr (kMma) {
    for (int i = tid; i < R * D; i += blockDim.x) refb[i] = Rh[i];
  } else {
    for (int i = tid; i < R * D; i += blockDim.x) refs[(i / D) * (D + 1) + i % D] = E::to_f(Rh[i]);
  }
  const bool keep32 = t.chunk_level == 1 && t.levels > 1;  // level 1 is the chunk level: keep fp32 values
  __syncthreads();
  const T* Kh = static_cast<const T*>(t.K) + size_t(h) * t.capacity * D;
  for (int64_t leaf = l0; leaf < l1; ++leaf) {
    for (int i = tid; i < b * VPR; i += blockDim.x)
      reinterpret_cast<uint4*>(keys)[i] = *reinterpret_cast<const uint4*>(Kh + size_t(leaf) * b * D + size_t(i) * (16 / sizeof(T)));
    __syncthreads();
    // the scores, the weights and the slopes exactly as the chunk kernel computes them
    if constexpr (kMma) scores_mma<D>(keys, D, b, refb, R, t.inv_sqrt_d, sc, tid >> 5, kAppendThreads / 32);
    else scores_fma<T, D>(keys, D, b, refs, R, t.inv_sqrt_d, sc);
    __syncthreads();
    for (int j = tid; j < R; j += blockDim.x) leaf_softmax(sc + j, R, b, &fg[j], &fg[kMaxRefs + j]);
    __syncthreads();
    T* rec = reinterpret_cast<T*>(t.rec(1, h, leaf));
    for (int i = tid; i < R * D; i += blockDim.x) {
      const int j = i / D, e = i % D;
      float acc = 0.f;
      for (int k = 0; k < b; ++k) acc = __fmaf_rn(sc[k * R + j], E::to_f(keys[size_t(k) * D + e]), acc);
      rec[size_t(j) * D + e] = E::from_f(acc);
      if (keep32) t.up(1, h, leaf)[size_t(j) * D + e] = acc;
    }
    float* bias = reinterpret_cast<float*>(t.rec(1, h, leaf) + size_t(R) * D * sizeof(T));
    const int padded = int((t.rec_bytes - size_t(R) * D * sizeof(T)) / 4);
    for (int j = tid; j < padded; j += blockDim.x) bias[j] = j < R ? __fsub_rn(fg[j], fg[kMaxRefs + j]) : 0.f;
    for (int j = tid; j < R; j += blockDim.x) {
      t.fval(1, h, leaf)[j] = fg[j];
      if (keep32) {
        float* u = t.up(1, h, leaf);
        u[size_t(R) * D + j] = fg[j];
        u[size_t(R) * D + R + j] = fg[kMaxRefs + j];
      }
    }
    __syncthreads();
  }
}

template <typename T, int D>
size_t append_fast_smem() {
  return size_t(kAppendMaxBlock) * D * sizeof(T) + size_t(kMaxRefs) * (D + 1) * 4 + size_t(kMaxRefs) * D * 2 +
         (size_t(kAppendMaxBlock) * kMaxRefs + 2 * kMaxRefs) * 4;
}


// Copy m new tokens ([Hkv][m][d] rows) into the cache at positions [n, n+m).
template <typename T, int D>
__global__ void append_copy_kernel(TreeDev t, const T* Knew, const T* Vnew, int64_t n, int64_t m) {
  constexpr int VPR = D * sizeof(T) / 16;
  const int64_t total = int64_t(t.hkv) * m * VPR;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t v = i % VPR, row = i / VPR;
    const int64_t h = row / m, r = row % m;
    const size_t src = size_t(row) * D + v * (16 / sizeof(T));
    const size_t dst = (size_t(h) * t.capacity + n + r) * D + v * (16 / sizeof(T));
    *reinterpret_cast<uint4*>(static_cast<T*>(t.K) + dst) = *reinterpret_cast<const uint4*>(Knew + src);
    *reinterpret_cast<uint4*>(static_cast<T*>(t.V) + dst) = *reinterpret_cast<const uint4*>(Vnew + src);
  }
}

// ------------------------------------------------------------------ host launchers
template <typename T, int D>
static cudaError_t launch_update_t(const TreeDev& t, int64_t n_old, int64_t n_new, cudaStream_t st,
                                   bool skip_chunk = false) {
  const int b = t.block, S = t.chunk_level;
  const int64_t CK = t.pow_b[S];
  const int64_t n1_old = n_old / b, n1_new = n_new / b;
  if (n1_new > n1_old && !skip_chunk) {
    const int64_t c0 = (n1_old * b) / CK;
    const int64_t c1 = (n1_new * b - 1) / CK;
    const ChunkSmem L = chunk_smem_layout<T, D>(b, S, t.refs);
    cudaError_t e = cudaFuncSetAttribute(chunk_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(L.total));
    if (e != cudaSuccess) return e;
    dim3 grid(unsigned(c1 - c0 + 1), unsigned(t.hkv));
    count_launches(1);
    chunk_kernel<T, D><<<grid, kBuildThreads, L.total, st>>>(t, n_new, n_old, c0);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  for (int level = S + 1; level <= t.levels; ++level) {
    const int64_t a0 = n_old / t.pow_b[level], a1 = n_new / t.pow_b[level];
    if (a1 <= a0) continue;
    const size_t sm = (size_t(b) * t.refs + 2 * t.refs) * 4;
    cudaError_t e = cudaFuncSetAttribute(upper_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm));
    if (e != cudaSuccess) return e;
    dim3 grid(unsigned(a1 - a0), unsigned(t.hkv));
    count_launches(1);
    upper_kernel<T, D><<<grid, kBuildThreads, sm, st>>>(t, level, a0);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (t.planes == ZHA_PLANES_FP4) {  // the router copies of the nodes this call completed
    for (int level = 1; level <= t.levels; ++level) {
      const int64_t a0 = n_old / t.pow_b[level], a1 = n_new / t.pow_b[level];
      if (a1 <= a0) continue;
      dim3 grid(unsigned(a1 - a0), unsigned(t.hkv));
      count_launches(1);
      quant4_kernel<T, D><<<grid, 128, 0, st>>>(t, level, a0);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  return cudaSuccess;
}

cudaError_t launch_tree_update(const TreeDev& t, int dtype, int64_t n_old, int64_t n_new, cudaStream_t st) {
  if (dtype == ZHA_BF16) {
    return t.d == 128 ? launch_update_t<__nv_bfloat16, 128>(t, n_old, n_new, st)
                      : launch_update_t<__nv_bfloat16, 64>(t, n_old, n_new, st);
  }
  return t.d == 128 ? launch_update_t<float, 128>(t, n_old, n_new, st) : launch_update_t<float, 64>(t, n_old, n_new, st);
}

// Whether an append of m tokens at n can take append_fast_kernel: no node of levels 2..S completes, the
// leaves fit its staging, and the copy is small.
bool append_fast_ok(const TreeDev& t, int64_t n, int64_t m) {
  if (t.block > kAppendMaxBlock || m > 64) return false;
  for (int level = 2; level <= t.chunk_level; ++level)
    if ((n + m) / t.pow_b[level] != n / t.pow_b[level]) return false;
  return true;
}

template <typename T, int D>
static cudaError_t launch_update_t(const TreeDev& t, int64_t n_old, int64_t n_new, cudaStream_t st, bool skip_chunk);

template <typename T, int D>
static cudaError_t launch_append_fast_t(const TreeDev& t, const void* Kn, const void* Vn, int64_t n, int64_t m,
                                        cudaStream_t st) {
  const size_t sm = append_fast_smem<T, D>();
  cudaError_t e = cudaFuncSetAttribute(append_fast_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm));
  if (e != cudaSuccess) return e;
  count_launches(1);
  append_fast_kernel<T, D><<<unsigned(t.hkv), kAppendThreads, sm, st>>>(t, static_cast<const T*>(Kn),
                                                                         static_cast<const T*>(Vn), n, m);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // levels above the chunk level that the new leaves complete, and FP4 router copies
  return launch_update_t<T, D>(t, n, n + m, st, /*skip_chunk=*/true);
}

cudaError_t launch_append_fast(const TreeDev& t, int dtype, const void* Kn, const void* Vn, int64_t n, int64_t m,
                               cudaStream_t st) {
  if (dtype == ZHA_BF16)
    return t.d == 128 ? launch_append_fast_t<__nv_bfloat16, 128>(t, Kn, Vn, n, m, st)
                      : launch_append_fast_t<__nv_bfloat16, 64>(t, Kn, Vn, n, m, st);
  return t.d == 128 ? launch_append_fast_t<float, 128>(t, Kn, Vn, n, m, st)
                    : launch_append_fast_t<float, 64>(t, Kn, Vn, n, m, st);
}

cudaError_t launch_append_copy(const TreeDev& t, int dtype, const void* Kn, const void* Vn, int64_t n, int64_t m,
                               cudaStream_t st) {
  const int64_t vecs = int64_t(t.hkv) * m * (t.d * (dtype == ZHA_BF16 ? 2 : 4) / 16);
  const int threads = 256;
  const unsigned blocks = unsigned(min64((vecs + threads - 1) / threads, 148 * 8));
  if (blocks == 0) return cudaSuccess;
  count_launches(1);
  if (dtype == ZHA_BF16) {
    if (t.d == 128)
      append_copy_kernel<__nv_bfloat16, 128><<<blocks, threads, 0, st>>>(
          t, static_cast<const __nv_bfloat16*>(Kn), static_cast<const __nv_bfloat16*>(Vn), n, m);
    else
      append_copy_kernel<__nv_bfloat16, 64><<<blocks, threads, 0, st>>>(
          t, static_cast<const __nv_bfloat16*>(Kn), static_cast<const __nv_bfloat16*>(Vn), n, m);
  } else {
    if (t.d == 128)
      append_copy_kernel<float, 128><<<blocks, threads, 0, st>>>(t, static_cast<const float*>(Kn),
                                                                  static_cast<const float*>(Vn), n, m);
    else
      append_copy_kernel<float, 64><<<blocks, threads, 0, st>>>(t, static_cast<const float*>(Kn),
                                                                 static_cast<const float*>(Vn), n, m);
  }
  return cudaGetLastError();
}

size_t chunk_smem_bytes(int dtype, int d, int block, int chunk_level, int R) {
  if (dtype == ZHA_BF16)
    return d == 128 ? chunk_smem_layout<__nv_bfloat16, 128>(block, chunk_level, R).total
                    : chunk_smem_layout<__nv_bfloat16, 64>(block, chunk_level, R).total;
  return d == 128 ? chunk_smem_layout<float, 128>(block, chunk_level, R).total
                  : chunk_smem_layout<float, 64>(block, chunk_level, R).total;
}

}  // namespace zha
