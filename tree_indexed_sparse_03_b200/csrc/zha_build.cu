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
#include "zha_args.cuh"

namespace zha {

constexpr int kBuildThreads = 256;

struct ChunkSmem {
  int CK, KS, RG, NN;
  size_t keys, refs, w, mu, fs, gs, total;
};

template <typename T, int D>
__host__ __device__ inline ChunkSmem chunk_smem_layout(int block, int chunk_level, int R) {
  ChunkSmem L;
  int CK = 1;
  for (int i = 0; i < chunk_level; ++i) CK *= block;
  L.CK = CK;
  L.KS = D + 16 / int(sizeof(T));  // key row stride in elements (16-byte pad)
  L.RG = R < 4 ? R : 4;
  int nn = 0, w = CK;
  for (int l = 1; l <= chunk_level; ++l) { w /= block; nn += w; }
  L.NN = nn;
  size_t off = 0;
  L.keys = off; off += size_t(CK) * L.KS * sizeof(T); off = (off + 15) & ~size_t(15);
  L.refs = off; off += size_t(R) * (D + 1) * 4;
  L.w = off;    off += size_t(CK) * L.RG * 4;
  L.mu = off;   off += size_t(nn) * L.RG * D * 4;
  L.fs = off;   off += size_t(nn) * L.RG * 4;
  L.gs = off;   off += size_t(nn) * L.RG * 4;
  L.total = (off + 15) & ~size_t(15);
  return L;
}

// One CTA per (chunk, KV head).  Computes every complete node of levels
// 1..S inside the chunk and writes those with index >= the previous count.
template <typename T, int D>
__global__ void __launch_bounds__(kBuildThreads) chunk_kernel(TreeDev t, int64_t n_tokens,
                                                              int64_t n_old, int64_t chunk0) {
  using E = Elem<T>;
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
  const int tid = threadIdx.x;

  extern __shared__ __align__(16) unsigned char smem[];
  T* keys = reinterpret_cast<T*>(smem + L.keys);
  float* refs = reinterpret_cast<float*>(smem + L.refs);
  float* w = reinterpret_cast<float*>(smem + L.w);
  float* mu = reinterpret_cast<float*>(smem + L.mu);
  float* fs = reinterpret_cast<float*>(smem + L.fs);
  float* gs = reinterpret_cast<float*>(smem + L.gs);

  // Stage the chunk's complete keys (16-byte vectors) and the fp32 refs.
  {
    constexpr int VPR = D * sizeof(T) / 16;  // vectors per key row
    const T* Kh = static_cast<const T*>(t.K) + (size_t(h) * t.capacity + key0) * D;
    for (int i = tid; i < nkeys * VPR; i += blockDim.x) {
      const int k = i / VPR, v = i % VPR;
      uint4 x = ldg_stream(Kh + size_t(k) * D + v * (16 / sizeof(T)));
      *reinterpret_cast<uint4*>(keys + size_t(k) * KS + v * (16 / sizeof(T))) = x;
    }
    const T* Rh = static_cast<const T*>(t.refsp) + size_t(h) * R * D;
    for (int i = tid; i < R * D; i += blockDim.x) refs[(i / D) * (D + 1) + i % D] = E::to_f(Rh[i]);
  }
  __syncthreads();

  // node slot of (level, index-in-chunk) inside the per-chunk arrays: level l starts at slot_off[l]
  int slot_off[kMaxLevels + 1];
  {
    int off = 0, wdt = CK;
    for (int l = 1; l <= S; ++l) {
      slot_off[l] = off;
      wdt /= b;
      off += wdt;
    }
  }
  auto slot = [&](int level, int i) { return slot_off[level] + i; };
  // loops over (node, reference query) rows of D values: thread tid takes element e of rows
  // tid / D, tid / D + RPI, ... (one division per row, none per element)
  constexpr int RPI = kBuildThreads / D;
  const int e_t = tid % D;

  int64_t pw = 1;
  for (int j0 = 0; j0 < R; j0 += RG) {
    const int rg = min(RG, R - j0);
    // scores s[k][jj]: sequential fma over the dimensions (keys read as 16-byte vectors)
    for (int i = tid; i < nkeys * rg; i += blockDim.x) {
      const int k = i / rg, jj = i - (i / rg) * rg;
      const T* kr = keys + size_t(k) * KS;
      const float* rr = refs + (j0 + jj) * (D + 1);
      constexpr int EPV = 16 / sizeof(T);
      float acc = 0.f;
#pragma unroll 2
      for (int e0 = 0; e0 < D; e0 += EPV) {
        float x[EPV];
        unpack16<T>(*reinterpret_cast<const uint4*>(kr + e0), x);
#pragma unroll
        for (int q = 0; q < EPV; ++q) acc = __fmaf_rn(x[q], rr[e0 + q], acc);
      }
      w[k * RG + jj] = __fmul_rn(acc, t.inv_sqrt_d);
    }
    __syncthreads();
    // leaf value, projected mean score and softmax weights
    for (int i = tid; i < nleaves * rg; i += blockDim.x) {
      const int li = i / rg, jj = i % rg;
      float* s = w + (li * b) * RG + jj;
      float m = -INFINITY;
      for (int k = 0; k < b; ++k) m = fmaxf(m, s[k * RG]);
      float Z = 0.f;
      for (int k = 0; k < b; ++k) Z = __fadd_rn(Z, expf(__fsub_rn(s[k * RG], m)));
      const float f = __fadd_rn(m, logf(Z));
      float g = 0.f;
      for (int k = 0; k < b; ++k) {
        const float wk = __fdiv_rn(expf(__fsub_rn(s[k * RG], m)), Z);
        g = __fmaf_rn(wk, s[k * RG], g);
        s[k * RG] = wk;
      }
      fs[slot(1, li) * RG + jj] = f;
      gs[slot(1, li) * RG + jj] = g;
    }
    __syncthreads();
    // leaf slopes mu
    for (int row = tid / D; row < nleaves * rg; row += RPI) {
      const int li = row / rg, jj = row - li * rg, e = e_t;
      float acc = 0.f;
      for (int k = 0; k < b; ++k)
        acc = __fmaf_rn(w[(li * b + k) * RG + jj], E::to_f(keys[size_t(li * b + k) * KS + e]), acc);
      mu[(size_t(slot(1, li)) * RG + jj) * D + e] = acc;
    }
    __syncthreads();
    // exact merges of levels 2..S inside the chunk
    int64_t bl = b;  // b^(level-1)
    for (int level = 2; level <= S; ++level) {
      bl *= b;
      const int64_t per_chunk = CK / bl;
      const int nval = int(min64(per_chunk, n_tokens / bl - chunk * per_chunk));
      if (nval > 0) {
        for (int i = tid; i < nval * rg; i += blockDim.x) {
          const int ni = i / rg, jj = i % rg;
          const int c0 = slot(level - 1, ni * b);
          float m = -INFINITY;
          for (int c = 0; c < b; ++c) m = fmaxf(m, fs[(c0 + c) * RG + jj]);
          float Z = 0.f;
          for (int c = 0; c < b; ++c) Z = __fadd_rn(Z, expf(__fsub_rn(fs[(c0 + c) * RG + jj], m)));
          const float f = __fadd_rn(m, logf(Z));
          float g = 0.f;
          for (int c = 0; c < b; ++c) {
            const float a = __fdiv_rn(expf(__fsub_rn(fs[(c0 + c) * RG + jj], m)), Z);
            w[(ni * b + c) * RG + jj] = a;
            g = __fmaf_rn(a, gs[(c0 + c) * RG + jj], g);
          }
          fs[slot(level, ni) * RG + jj] = f;
          gs[slot(level, ni) * RG + jj] = g;
        }
        __syncthreads();
        for (int row = tid / D; row < nval * rg; row += RPI) {
          const int ni = row / rg, jj = row - ni * rg, e = e_t;
          const int c0 = slot(level - 1, ni * b);
          float acc = 0.f;
          for (int c = 0; c < b; ++c)
            acc = __fmaf_rn(w[(ni * b + c) * RG + jj], mu[(size_t(c0 + c) * RG + jj) * D + e], acc);
          mu[(size_t(slot(level, ni)) * RG + jj) * D + e] = acc;
        }
      }
      __syncthreads();
    }
    // write the nodes that are new in this call
    pw = 1;
    for (int level = 1; level <= S; ++level) {
      pw *= b;
      const int64_t per_chunk = CK / pw;
      const int64_t base = chunk * per_chunk;
      const int nval = int(min64(per_chunk, n_tokens / pw - base));
      const int64_t first_new = n_old / pw;
      const bool keep32 = (level == S) && (S < t.levels);
      for (int row = tid / D; row < nval * rg; row += RPI) {
        const int ni = row / rg, jj = row - ni * rg, e = e_t;
        const int64_t gi = base + ni;
        if (gi < first_new) continue;
        const float v = mu[(size_t(slot(level, ni)) * RG + jj) * D + e];
        T* rec = reinterpret_cast<T*>(t.rec(level, h, gi));
        rec[size_t(j0 + jj) * D + e] = E::from_f(v);
        if (keep32) t.up(level, h, gi)[size_t(j0 + jj) * D + e] = v;
      }
      for (int i = tid; i < nval * rg; i += blockDim.x) {
        const int jj = i % rg, ni = i / rg;
        const int64_t gi = base + ni;
        if (gi < first_new) continue;
        const float f = fs[slot(level, ni) * RG + jj];
        const float g = gs[slot(level, ni) * RG + jj];
        float* bias = reinterpret_cast<float*>(t.rec(level, h, gi) + size_t(R) * D * sizeof(T));
        bias[j0 + jj] = __fsub_rn(f, g);
        t.fval(level, h, gi)[j0 + jj] = f;
        if (keep32) {
          float* u = t.up(level, h, gi);
          u[size_t(R) * D + j0 + jj] = f;
          u[size_t(R) * D + R + j0 + jj] = g;
        }
      }
    }
    __syncthreads();
  }
  // zero the padding after bias[R] once per new node so records are fully defined
  {
    pw = 1;
    const int pad = int((t.rec_bytes - size_t(R) * D * sizeof(T)) / 4) - R;
    if (pad > 0) {
      for (int level = 1; level <= S; ++level) {
        pw *= b;
        const int64_t per_chunk = CK / pw, base = chunk * per_chunk;
        const int nval = int(min64(per_chunk, n_tokens / pw - base));
        const int64_t first_new = n_old / pw;
        for (int i = tid; i < nval * pad; i += blockDim.x) {
          const int64_t gi = base + i / pad;
          if (gi < first_new) continue;
          reinterpret_cast<float*>(t.rec(level, h, gi) + size_t(R) * D * sizeof(T))[R + i % pad] = 0.f;
        }
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
  constexpr int VPR = D * sizeof(T) / 16;
  const int h = blockIdx.x, tid = threadIdx.x;
  const int b = t.block, R = t.refs;
  extern __shared__ __align__(16) unsigned char smem[];
  float* refs = reinterpret_cast<float*>(smem);                      // [R][D + 1]
  float* sc = refs + size_t(R) * (D + 1);                             // [b][R] scores, then weights
  float* fg = sc + size_t(kAppendMaxBlock) * kMaxRefs;                // [R] f, [R] g
  T* keys = reinterpret_cast<T*>(fg + 2 * kMaxRefs);                   // [b][D]
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
  for (int i = tid; i < R * D; i += blockDim.x) refs[(i / D) * (D + 1) + i % D] = E::to_f(Rh[i]);
  const bool keep32 = t.chunk_level == 1 && t.levels > 1;  // level 1 is the chunk level: keep fp32 values
  __syncthreads();
  const T* Kh = static_cast<const T*>(t.K) + size_t(h) * t.capacity * D;
  for (int64_t leaf = l0; leaf < l1; ++leaf) {
    for (int i = tid; i < b * D; i += blockDim.x) keys[i] = Kh[size_t(leaf) * b * D + i];
    __syncthreads();
    // scores s[k][j] = (r_j . k) / sqrt(d): sequential fma over the dimensions
    for (int i = tid; i < b * R; i += blockDim.x) {
      const int k = i / R, j = i % R;
      const T* kr = keys + size_t(k) * D;
      const float* rr = refs + j * (D + 1);
      float acc = 0.f;
#pragma unroll 8
      for (int e = 0; e < D; ++e) acc = __fmaf_rn(E::to_f(kr[e]), rr[e], acc);
      sc[k * kMaxRefs + j] = __fmul_rn(acc, t.inv_sqrt_d);
    }
    __syncthreads();
    // value, projected mean score and softmax weights of each reference query
    for (int j = tid; j < R; j += blockDim.x) {
      float mx = -INFINITY;
      for (int k = 0; k < b; ++k) mx = fmaxf(mx, sc[k * kMaxRefs + j]);
      float Z = 0.f;
      for (int k = 0; k < b; ++k) Z = __fadd_rn(Z, expf(__fsub_rn(sc[k * kMaxRefs + j], mx)));
      const float f = __fadd_rn(mx, logf(Z));
      float g = 0.f;
      for (int k = 0; k < b; ++k) {
        const float wk = __fdiv_rn(expf(__fsub_rn(sc[k * kMaxRefs + j], mx)), Z);
        g = __fmaf_rn(wk, sc[k * kMaxRefs + j], g);
        sc[k * kMaxRefs + j] = wk;
      }
      fg[j] = f;
      fg[kMaxRefs + j] = g;
    }
    __syncthreads();
    // slopes mu, the record (mu in the element type, intercepts), f, and the fp32 copy at the chunk level
    T* rec = reinterpret_cast<T*>(t.rec(1, h, leaf));
    for (int i = tid; i < R * D; i += blockDim.x) {
      const int j = i / D, e = i % D;
      float acc = 0.f;
      for (int k = 0; k < b; ++k) acc = __fmaf_rn(sc[k * kMaxRefs + j], E::to_f(keys[size_t(k) * D + e]), acc);
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
  return (size_t(kMaxRefs) * (D + 1) + size_t(kAppendMaxBlock) * kMaxRefs + 2 * kMaxRefs) * 4 +
         size_t(kAppendMaxBlock) * D * sizeof(T);
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
