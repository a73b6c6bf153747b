// Fused ZHA decode: top-down top-p routing over the tree, then sparse
// softmax attention over the kept blocks, the sink and the tail.
//
// Method ("Zyphra Hierarchical Attention", Zyphra blog, section "Routing in
// the tree"; tanhow.com summary, section "How does top-p routing choose
// tokens?"): the query scores the top-level summaries, keeps the smallest set
// covering estimated attention mass p, expands only the kept nodes' children,
// and repeats until it reaches raw KV entries; ordinary attention then runs on
// the selected keys, with the first token always kept as attention sink.  The
// estimate of a node is the maximum of its tangent planes,
// e(q) = max_j (b_j + q.mu_j/sqrt(d)) (summary, section "Building the tree").
// Readings where the pages are silent: the first candidate set is the complete
// top nodes plus the roots of the partial subtrees; "reaching p" is cumulative
// mass >= p; ties in e go to the lower start token; tokens after the last
// complete block (the tail) are always attended.
//
// GPU design.  One thread-block cluster of CS CTAs per (sequence, query head);
// the whole decode of that head is one kernel launch with one cluster barrier
// per routing step:
//   score   each CTA scores the candidates it owns (the children of the kept
//           parents whose rank is = its cluster rank mod CS) with one warp per
//           node, and writes (descending key of e, node code) at the
//           candidate's canonical position in the step's global buffer;
//   barrier
//   select  every CTA reads the whole buffer and computes the same cut:
//           masses w = exp(e - max e) as 2^-40 fixed-point integers (exact,
//           order-independent sums), a 1024-bin histogram of the masses over
//           (max e - e) in 1/32-logit bins finds the bin holding the cut, and
//           the few entries of that bin are ordered by (e desc, start asc) to
//           find the last kept entry;  kept = every entry ordered at or before
//           it;  each CTA then takes its round-robin share of the kept
//           parents (next step) and of the kept leaves (attention).
// After the last step each CTA attends over its share of the kept blocks
// (plus the sink and tail on the last CTA) with an online softmax, and the
// partial (max, sum, output) triples are combined in CTA 0's shared memory
// over distributed shared memory.
#include <cooperative_groups.h>

#include "zha_args.cuh"

namespace cg = cooperative_groups;

namespace zha {

struct Entry {
  uint32_t key;   // desc_key(e)
  uint32_t code;  // node_code(level, index)
};

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kSelSmem = 4096;   // entries cached in shared memory
constexpr int kBins = 1024;
constexpr float kBinScale = 32.f;
constexpr int kMaxCluster = 16;

constexpr int kLeafSmem = 3840;  // leaf indices cached for the attention phase

struct AttendSmem {
  uint32_t leaf[kLeafSmem];
  float grp[kDecWarps * 4][2 + 128];  // per lane-group partials (m, l, o[d])
};

struct __align__(16) DecSmem {
  union {
    Entry cache[kSelSmem];            // routing: the step's candidate entries
    AttendSmem att;                   // attention: this CTA's leaf list + group partials
  };
  unsigned long long hist[kBins];
  unsigned long long cut_key[32];
  unsigned long long cut_w[32];
  float part[kMaxCluster][2 + 128];   // partials received by CTA 0 (m, l, o[d])
  unsigned long long red64[kDecWarps];
  uint32_t red32[kDecWarps * 2];
  unsigned long long bcast64[4];
  int bcast32[8];
};

__device__ __forceinline__ uint32_t root_code(const DecodeArgs& a, int64_t i) {
  const int L = a.t.levels, b = a.t.block;
  if (i < a.nl[L]) return node_code(L, uint32_t(i));
  int64_t r = i - a.nl[L];
  for (int l = L - 1; l >= 1; --l) {
    const int64_t cnt = a.nl[l] - int64_t(b) * a.nl[l + 1];
    if (r < cnt) return node_code(l, uint32_t(int64_t(b) * a.nl[l + 1] + r));
    r -= cnt;
  }
  return 0;
}

__device__ __forceinline__ uint64_t entry_key64(const DecodeArgs& a, Entry en) {
  const uint64_t start = uint64_t(code_index(en.code)) * uint64_t(a.t.pow_b[code_level(en.code)]);
  return (uint64_t(en.key) << 32) | start;
}

// ceil(p * Z) for p = mant * 2^-shift < 1, exactly (128-bit product).
__device__ __forceinline__ unsigned long long ceil_p_times(uint64_t Z, uint32_t mant, int shift) {
  const uint64_t lo = Z * uint64_t(mant);
  const uint64_t hi = __umul64hi(Z, uint64_t(mant));
  if (shift >= 128) return (lo | hi) ? 1ull : 0ull;
  uint64_t q, rem_nz;
  if (shift >= 64) {
    const int s = shift - 64;
    q = s ? (hi >> s) : hi;
    rem_nz = lo | (s ? (hi & ((1ull << s) - 1)) : 0ull);
  } else if (shift == 0) {
    q = lo;
    rem_nz = 0;
  } else {
    q = (lo >> shift) | (hi << (64 - shift));
    rem_nz = lo & ((1ull << shift) - 1);
  }
  return q + (rem_nz ? 1ull : 0ull);
}

// Estimate e(q) of one node, computed by a whole warp.  The lane's q slice
// covers elements [cl*EPC, cl*EPC+EPC) with cl = lane % CPR.
template <typename T, int D>
__device__ __forceinline__ float score_node(const TreeDev& t, int head, uint32_t code, const float* qs,
                                            int lane) {
  constexpr int EPC = 16 / sizeof(T);
  constexpr int CPR = D * sizeof(T) / 16;  // 16-byte chunks per ref row
  constexpr int RPI = 32 / CPR;            // refs per warp pass
  const int R = t.refs;
  const char* rec = t.rec(code_level(code), head, code_index(code));
  const float* bias = reinterpret_cast<const float*>(rec + size_t(R) * D * sizeof(T));
  const int sub = lane / CPR, cl = lane % CPR;
  float best = -INFINITY;
  constexpr int kBatch = 8;
  for (int j0 = 0; j0 < R; j0 += RPI * kBatch) {
    uint4 v[kBatch];
    float bj[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = j0 + u * RPI + sub;
      if (j < R) {
        v[u] = ldg_stream(rec + (size_t(j) * CPR + cl) * 16);
        bj[u] = __ldg(bias + j);
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = j0 + u * RPI + sub;
      float part = 0.f;
      if (j < R) {
        float x[EPC];
        unpack16<T>(v[u], x);
#pragma unroll
        for (int i = 0; i < EPC; ++i) part = fmaf(x[i], qs[i], part);
      }
#pragma unroll
      for (int off = CPR / 2; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      if (j < R) best = fmaxf(best, fmaf(part, t.inv_sqrt_d, bj[u]));
      if (j0 + (u + 1) * RPI >= R) break;
    }
  }
#pragma unroll
  for (int off = 16; off >= CPR; off >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, off));
  return best;
}

// Block-wide exclusive scan of one value per thread; returns the exclusive
// prefix and writes the block total to *total (all threads).
__device__ __forceinline__ uint32_t block_scan_u32(uint32_t v, uint32_t* red, uint32_t* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) red[wid] = x;
  __syncthreads();
  uint32_t base = 0, tot = 0;
  for (int w = 0; w < kDecWarps; ++w) {
    const uint32_t s = red[w];
    if (w < wid) base += s;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return base + x - v;
}

__device__ __forceinline__ unsigned long long block_scan_u64(unsigned long long v, unsigned long long* red,
                                                             unsigned long long* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) red[wid] = x;
  __syncthreads();
  unsigned long long base = 0, tot = 0;
  for (int w = 0; w < kDecWarps; ++w) {
    const unsigned long long s = red[w];
    if (w < wid) base += s;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return base + x - v;
}

__device__ __forceinline__ uint32_t block_min_u32(uint32_t v, uint32_t* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, off));
  if (lane == 0) red[wid] = v;
  __syncthreads();
  uint32_t m = 0xffffffffu;
  for (int w = 0; w < kDecWarps; ++w) m = min(m, red[w]);
  __syncthreads();
  return m;
}

__device__ __forceinline__ Entry load_entry(const Entry* E, int64_t i, bool cached, const DecSmem& sm) {
  if (cached) return sm.cache[i];
  const uint2 v = __ldcg(reinterpret_cast<const uint2*>(E + i));
  return Entry{v.x, v.y};
}

__device__ __forceinline__ int entry_bin(float m, uint32_t key) {
  const float x = __fsub_rn(m, desc_key_value(key));
  const float y = fminf(__fmul_rn(x, kBinScale), float(kBins - 1));
  return int(y);
}

__device__ __forceinline__ unsigned long long entry_mass(float m, uint32_t key) {
  const float w = expf(__fsub_rn(desc_key_value(key), m));
  return __float2ull_rn(w * 1099511627776.0f);  // 2^40
}

// The cut of one routing step: the largest 64-bit order key (e desc, start
// asc) that is kept.  Every thread returns the same value.
__device__ unsigned long long select_cut(const DecodeArgs& a, const Entry* E, int64_t n, bool cached,
                                         DecSmem& sm) {
  const int tid = threadIdx.x;
  uint32_t kmin = 0xffffffffu;
  for (int64_t i = tid; i < n; i += kDecThreads) kmin = min(kmin, load_entry(E, i, cached, sm).key);
  kmin = block_min_u32(kmin, sm.red32);
  if (a.p_all) return ~0ull;
  const float m = desc_key_value(kmin);

  for (int i = tid; i < kBins; i += kDecThreads) sm.hist[i] = 0ull;
  __syncthreads();
  for (int64_t i = tid; i < n; i += kDecThreads) {
    const Entry en = load_entry(E, i, cached, sm);
    atomicAdd(&sm.hist[entry_bin(m, en.key)], entry_mass(m, en.key));
  }
  __syncthreads();
  // prefix over the bins (kBins / kDecThreads consecutive bins per thread)
  constexpr int BPT = kBins / kDecThreads;
  unsigned long long local = 0;
#pragma unroll
  for (int k = 0; k < BPT; ++k) local += sm.hist[tid * BPT + k];
  unsigned long long Z;
  unsigned long long before = block_scan_u64(local, sm.red64, &Z);
  const unsigned long long T = ceil_p_times(Z, a.p_mant, a.p_shift);  // keep while mass before < T
  if (tid == 0) sm.bcast32[0] = -1;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < BPT; ++k) {
    const unsigned long long hb = sm.hist[tid * BPT + k];
    if (before < T && before + hb >= T) {
      sm.bcast32[0] = tid * BPT + k;
      sm.bcast64[0] = before;
    }
    before += hb;
  }
  __syncthreads();
  const int cb = sm.bcast32[0];
  const unsigned long long below = sm.bcast64[0];
  if (cb < 0) return ~0ull;  // cannot happen for 0 < p < 1; keep everything
  // gather the entries of the cut bin
  if (tid == 0) sm.bcast32[1] = 0;
  __syncthreads();
  for (int64_t i = tid; i < n; i += kDecThreads) {
    const Entry en = load_entry(E, i, cached, sm);
    if (entry_bin(m, en.key) == cb) {
      const int s = atomicAdd(&sm.bcast32[1], 1);
      if (s < 32) {
        sm.cut_key[s] = entry_key64(a, en);
        sm.cut_w[s] = entry_mass(m, en.key);
      }
    }
  }
  __syncthreads();
  const int cnt = sm.bcast32[1];
  if (cnt <= 32) {
    if (tid < 32) {
      unsigned long long k = tid < cnt ? sm.cut_key[tid] : ~0ull;
      unsigned long long w = tid < cnt ? sm.cut_w[tid] : 0ull;
      // bitonic sort of 32 (key asc), carrying w
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          const unsigned long long ok = __shfl_xor_sync(0xffffffffu, k, stride);
          const unsigned long long ow = __shfl_xor_sync(0xffffffffu, w, stride);
          const bool up = ((tid & size) == 0);
          const bool lower = ((tid & stride) == 0);
          const bool take_min = (up == lower);
          const bool swap = take_min ? (ok < k) : (ok > k);
          if (swap) { k = ok; w = ow; }
        }
      }
      unsigned long long c = w;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, c, off);
        if (tid >= off) c += y;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, tid < cnt && below + c >= T);
      const int first = hit ? __ffs(hit) - 1 : cnt - 1;
      const unsigned long long cut = __shfl_sync(0xffffffffu, k, first);
      if (tid == 0) sm.bcast64[1] = cut;
    }
    __syncthreads();
    return sm.bcast64[1];
  }
  // Many entries share the cut bin (ties or near-ties): radix select on the
  // 64-bit order key, 8 bits per pass, over the bin's entries.
  const unsigned long long target = T - below;  // > 0
  unsigned long long prefix = 0, acc_below = 0;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = tid; i < 256; i += kDecThreads) sm.hist[i] = 0ull;
    __syncthreads();
    for (int64_t i = tid; i < n; i += kDecThreads) {
      const Entry en = load_entry(E, i, cached, sm);
      if (entry_bin(m, en.key) != cb) continue;
      const unsigned long long k64 = entry_key64(a, en);
      if (pass > 0 && (k64 >> (shift + 8)) != (prefix >> (shift + 8))) continue;
      atomicAdd(&sm.hist[(k64 >> shift) & 255], entry_mass(m, en.key));
    }
    __syncthreads();
    if (tid == 0) {
      unsigned long long c = acc_below;
      int digit = 255;
      for (int dgt = 0; dgt < 256; ++dgt) {
        if (c + sm.hist[dgt] >= target) { digit = dgt; break; }
        c += sm.hist[dgt];
      }
      sm.bcast64[2] = prefix | (uint64_t(digit) << shift);
      sm.bcast64[3] = c;
    }
    __syncthreads();
    prefix = sm.bcast64[2];
    acc_below = sm.bcast64[3];
    __syncthreads();
  }
  return prefix;
}

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads, 3) decode_kernel(DecodeArgs a) {
  using E = Elem<T>;
  constexpr int EPC = 16 / sizeof(T);
  constexpr int CPR = D * sizeof(T) / 16;
  constexpr int KPW = 32 / CPR;  // keys per warp pass in the attention loop
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = int(cluster.num_blocks());
  const int r = int(cluster.block_rank());
  const int h = blockIdx.y, bb = blockIdx.z;
  const int kvh = h / a.t.group;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int b = a.t.block;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>(smem_raw);

  char* ws = a.ws + uint64_t(bb * a.t.hq + h) * a.ws_per_bh;
  Entry* sel[2] = {reinterpret_cast<Entry*>(ws), reinterpret_cast<Entry*>(ws) + a.cap_sel};
  const int64_t per_cta = a.cap_list / CS;
  uint2* my_par = reinterpret_cast<uint2*>(ws + 2 * a.cap_sel * sizeof(Entry)) + r * per_cta;
  uint32_t* my_leaf = reinterpret_cast<uint32_t*>(ws + 2 * a.cap_sel * sizeof(Entry) + a.cap_list * 8) + r * per_cta;

  // the lane's slice of q (fp32)
  float qs[EPC];
  {
    const T* q = static_cast<const T*>(a.Q) + (size_t(bb) * a.t.hq + h) * D + (lane % CPR) * EPC;
    const uint4 v = *reinterpret_cast<const uint4*>(q);
    unpack16<T>(v, qs);
  }

  // distributed shared memory of CTA 0 is written at the end: make sure every
  // CTA of the cluster has started when no routing step provides a barrier
  if (a.n_steps == 0) cluster.sync();

  int64_t n_cand = a.n_roots;
  int64_t my_npar = 0;          // parents this CTA expands in the next step
  int64_t leafbase = 0;         // kept leaves so far (all CTAs)
  int64_t scored = 0;
  bool leaf0 = false;
  int steps_taken = 0;

  for (int step = 0; step < a.n_steps; ++step) {
    Entry* S = sel[step & 1];
    // ---- score the candidates this CTA owns
    if (step == 0) {
      for (int64_t i = r + int64_t(CS) * wid; i < n_cand; i += int64_t(CS) * kDecWarps) {
        const uint32_t code = root_code(a, i);
        const float e = score_node<T, D>(a.t, kvh, code, qs, lane);
        if (lane == 0) S[i] = Entry{desc_key(e), code};
      }
    } else {
      const int64_t items = my_npar * b;
      for (int64_t u = wid; u < items; u += kDecWarps) {
        const uint2 pr = __ldcg(my_par + u / b);
        const int c = int(u % b);
        const uint32_t pc = pr.x;
        const uint32_t code = node_code(code_level(pc) - 1, code_index(pc) * uint32_t(b) + uint32_t(c));
        const float e = score_node<T, D>(a.t, kvh, code, qs, lane);
        const int64_t pos = int64_t(pr.y) * b + c;
        if (lane == 0) {
          if (pos < a.cap_sel) S[pos] = Entry{desc_key(e), code};
          else raise_status(a.t.status, ZHA_ERR_CAPACITY);
        }
      }
    }
    __threadfence();
    cluster.sync();
    if (n_cand == 0) continue;   // uniform across the cluster
    ++steps_taken;

    // ---- select (identical in every CTA of the cluster)
    const bool cached = n_cand <= kSelSmem;
    if (cached) {
      for (int64_t i = tid; i < n_cand; i += kDecThreads) {
        const uint2 v = __ldcg(reinterpret_cast<const uint2*>(S + i));
        sm.cache[i] = Entry{v.x, v.y};
      }
      __syncthreads();
    }
    if (a.scored && r == 0) {
      int32_t* out = a.scored + (size_t(bb) * a.t.hq + h) * a.scored_cap;
      for (int64_t i = tid; i < n_cand; i += kDecThreads)
        if (scored + i < a.scored_cap) out[scored + i] = int32_t(load_entry(S, i, cached, sm).code);
    }
    scored += n_cand;
    const unsigned long long cut = select_cut(a, S, n_cand, cached, sm);

    // ---- ranks of the kept entries in canonical order
    const int64_t per_thr = (n_cand + kDecThreads - 1) / kDecThreads;
    const int64_t lo = min64(n_cand, tid * per_thr), hi = min64(n_cand, lo + per_thr);
    uint32_t nleaf = 0, npar = 0;
    for (int64_t i = lo; i < hi; ++i) {
      const Entry en = load_entry(S, i, cached, sm);
      if (entry_key64(a, en) <= cut) {
        if (code_level(en.code) == 1) ++nleaf; else ++npar;
      }
    }
    uint32_t tot_leaf, tot_par;
    uint32_t leaf_rank = block_scan_u32(nleaf, sm.red32, &tot_leaf);
    uint32_t par_rank = block_scan_u32(npar, sm.red32, &tot_par);
    for (int64_t i = lo; i < hi; ++i) {
      const Entry en = load_entry(S, i, cached, sm);
      if (entry_key64(a, en) > cut) continue;
      if (code_level(en.code) == 1) {
        const int64_t g = leafbase + leaf_rank++;
        if (code_index(en.code) == 0) leaf0 = true;
        if (g % CS == r) {
          const int64_t slot = g / CS;
          if (slot < per_cta) my_leaf[slot] = code_index(en.code);
          else raise_status(a.t.status, ZHA_ERR_CAPACITY);
        }
        if (a.kept && r == 0 && g < a.kept_stride)
          a.kept[(size_t(bb) * a.t.hq + h) * a.kept_stride + g] = int32_t(code_index(en.code));
      } else {
        const uint32_t pr = par_rank++;
        if (int(pr % CS) == r) {
          const int64_t slot = pr / CS;
          if (slot < per_cta) my_par[slot] = make_uint2(en.code, pr);
          else raise_status(a.t.status, ZHA_ERR_CAPACITY);
        }
      }
    }
    // every CTA learns whether leaf 0 was kept (a leaf-0 entry may sit in another thread's range)
    leaf0 = __syncthreads_or(leaf0);
    leafbase += tot_leaf;
    my_npar = min64((int64_t(tot_par) > r) ? (int64_t(tot_par) - r + CS - 1) / CS : 0, per_cta);
    n_cand = int64_t(tot_par) * b;
    if (n_cand > a.cap_sel) {
      raise_status(a.t.status, ZHA_ERR_CAPACITY);
      n_cand = a.cap_sel;
      my_npar = 0;
    }
  }

  // ---- attention over this CTA's share of the attended tokens
  const int64_t n1 = a.nl[1];
  const int64_t my_nleaf = (leafbase > r) ? (leafbase - r + CS - 1) / CS : 0;
  const int64_t my_leaf_keys = min64(my_nleaf, per_cta) * b;
  int64_t extra0 = 0, extra_cnt = 0;  // [extra0, extra0+extra_cnt) after an optional sink
  bool sink = false;
  if (r == CS - 1) {
    sink = (n1 > 0) && !leaf0;
    extra0 = n1 * b;
    extra_cnt = a.n_tokens - n1 * b;
  }
  const int64_t total = my_leaf_keys + (sink ? 1 : 0) + extra_cnt;
  // cache this CTA's leaf list in shared memory (the entry cache is free now)
  uint32_t* leaf_s = sm.att.leaf;
  const int64_t nls = min64(my_leaf_keys / b, int64_t(kLeafSmem));
  __syncthreads();
  for (int64_t i = tid; i < nls; i += kDecThreads) leaf_s[i] = __ldcg(my_leaf + i);
  __syncthreads();

  const T* Kh = static_cast<const T*>(a.t.K) + size_t(kvh) * a.t.capacity * D;
  const T* Vh = static_cast<const T*>(a.t.V) + size_t(kvh) * a.t.capacity * D;
  const int sub = lane / CPR, cl = lane % CPR;
  float m_run = -INFINITY, l_run = 0.f;
  float o[EPC];
#pragma unroll
  for (int i = 0; i < EPC; ++i) o[i] = 0.f;
  constexpr int kU = 4;
  const int64_t gstride = int64_t(kDecWarps) * KPW;
  // the loop bound is warp-uniform (wb); lane groups differ only through `ok`
  for (int64_t wb = int64_t(wid) * KPW; wb < total; wb += gstride * kU) {
    uint4 kv[kU], vv[kU];
    bool ok[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t idx = wb + sub + u * gstride;
      ok[u] = idx < total;
      if (ok[u]) {
        int64_t tok;
        if (idx < my_leaf_keys) {
          const int64_t li = idx / b;
          const uint32_t leaf = li < nls ? leaf_s[li] : __ldcg(my_leaf + li);
          tok = int64_t(leaf) * b + idx % b;
        } else {
          int64_t x = idx - my_leaf_keys;
          if (sink) {
            if (x == 0) tok = 0;
            else tok = extra0 + x - 1;
          } else {
            tok = extra0 + x;
          }
        }
        kv[u] = ldg_stream(Kh + size_t(tok) * D + cl * EPC);
        vv[u] = ldg_stream(Vh + size_t(tok) * D + cl * EPC);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      float kx[EPC];
      float s = 0.f;
      if (ok[u]) {
        unpack16<T>(kv[u], kx);
#pragma unroll
        for (int i = 0; i < EPC; ++i) s = fmaf(kx[i], qs[i], s);
      }
#pragma unroll
      for (int off = CPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      if (ok[u]) {
        s *= a.t.inv_sqrt_d;
        const float mn = fmaxf(m_run, s);
        const float sc = expf(m_run - mn);
        const float pk = expf(s - mn);
        l_run = l_run * sc + pk;
        float vx[EPC];
        unpack16<T>(vv[u], vx);
#pragma unroll
        for (int i = 0; i < EPC; ++i) o[i] = fmaf(pk, vx[i], o[i] * sc);
        m_run = mn;
      }
    }
  }
  // lane-group partials -> shared memory
  const int grp = wid * KPW + sub;
  if (cl == 0) {
    sm.att.grp[grp][0] = m_run;
    sm.att.grp[grp][1] = l_run;
  }
#pragma unroll
  for (int i = 0; i < EPC; ++i) sm.att.grp[grp][2 + cl * EPC + i] = o[i];
  __syncthreads();
  // CTA partial: combine the groups in a fixed order; send it to CTA 0
  float* dst = cluster.map_shared_rank(&sm.part[0][0], 0) + r * (2 + 128);
  {
    float M = -INFINITY;
    for (int g = 0; g < kDecWarps * KPW; ++g) M = fmaxf(M, sm.att.grp[g][0]);
    for (int e = tid; e < D + 1; e += kDecThreads) {
      float acc = 0.f;
      for (int g = 0; g < kDecWarps * KPW; ++g) {
        const float mg = sm.att.grp[g][0];
        if (mg == -INFINITY) continue;
        const float sc = expf(mg - M);
        acc = fmaf(sc, e == 0 ? sm.att.grp[g][1] : sm.att.grp[g][1 + e], acc);
      }
      dst[1 + e] = acc;   // dst[1] = l, dst[2 + i] = o[i]
    }
    if (tid == 0) dst[0] = M;
  }
  cluster.sync();
  if (r == 0) {
    float M = -INFINITY;
    for (int c = 0; c < CS; ++c) M = fmaxf(M, sm.part[c][0]);
    float lsum = 0.f;
    for (int c = 0; c < CS; ++c)
      if (sm.part[c][0] != -INFINITY) lsum = fmaf(expf(sm.part[c][0] - M), sm.part[c][1], lsum);
    const float inv = 1.f / lsum;
    float* out = a.O + (size_t(bb) * a.t.hq + h) * D;
    for (int e = tid; e < D; e += kDecThreads) {
      float acc = 0.f;
      for (int c = 0; c < CS; ++c)
        if (sm.part[c][0] != -INFINITY) acc = fmaf(expf(sm.part[c][0] - M), sm.part[c][2 + e], acc);
      out[e] = acc * inv;
    }
    if (tid == 0) {
      if (a.kept_cnt) a.kept_cnt[bb * a.t.hq + h] = int32_t(leafbase);
      if (a.stats) {
        int64_t* st = a.stats + (size_t(bb) * a.t.hq + h) * ZHA_STAT_COUNT;
        st[ZHA_STAT_NODES_SCORED] = scored;
        st[ZHA_STAT_LEAVES_KEPT] = leafbase;
        st[ZHA_STAT_KEYS] = leafbase * b + ((n1 > 0 && !leaf0) ? 1 : 0) + (a.n_tokens - n1 * b);
        st[ZHA_STAT_STEPS] = steps_taken;
      }
    }
  }
}

// ------------------------------------------------------------------ host launcher
template <typename T, int D>
static cudaError_t launch_decode_t(const DecodeArgs& a, int B, int cs, cudaStream_t st) {
  auto kern = decode_kernel<T, D>;
  const size_t smem = sizeof(DecSmem);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  if (cs > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(cs), unsigned(a.t.hq), unsigned(B));
  cfg.blockDim = dim3(kDecThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = unsigned(cs);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launches(1);
  return cudaLaunchKernelEx(&cfg, kern, a);
}

// Largest usable cluster size <= want (a power of two) for this kernel.
template <typename T, int D>
static int usable_cluster_t(int want) {
  auto kern = decode_kernel<T, D>;
  const size_t smem = sizeof(DecSmem);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess) return 0;
  cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  for (int cs = want; cs >= 1; cs >>= 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(cs), 1, 1);
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(cs);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) == cudaSuccess && nclusters > 0) return cs;
    cudaGetLastError();
  }
  return 0;
}

cudaError_t launch_decode(const DecodeArgs& a, int dtype, int B, int cs, cudaStream_t st) {
  if (dtype == ZHA_BF16)
    return a.t.d == 128 ? launch_decode_t<__nv_bfloat16, 128>(a, B, cs, st)
                        : launch_decode_t<__nv_bfloat16, 64>(a, B, cs, st);
  return a.t.d == 128 ? launch_decode_t<float, 128>(a, B, cs, st) : launch_decode_t<float, 64>(a, B, cs, st);
}

int usable_cluster(int dtype, int d, int want) {
  if (dtype == ZHA_BF16) return d == 128 ? usable_cluster_t<__nv_bfloat16, 128>(want) : usable_cluster_t<__nv_bfloat16, 64>(want);
  return d == 128 ? usable_cluster_t<float, 128>(want) : usable_cluster_t<float, 64>(want);
}

size_t decode_smem_bytes() { return sizeof(DecSmem); }

}  // namespace zha
