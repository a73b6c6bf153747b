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
// GPU design.  One persistent cooperative launch per decode call; all query
// heads of all sequences are routed together so that the whole GPU shares
// the work of the heads whose routing is diffuse.  Phases are separated by a
// software grid barrier (a monotonic arrival counter; bounded spin: on
// timeout the kernel raises ZHA_ERR_TIMEOUT and returns):
//   score   (all CTAs) the step's candidates of every head form one list that
//           is cut into contiguous per-warp ranges; each warp streams the node
//           records of its range through a ring of shared-memory slots with
//           cp.async (several records in flight per warp), computes the
//           estimates in fp32 and writes (descending key of e, node code) at
//           the candidate's position in its head's step buffer;
//   select  (one CTA per head) masses w = exp(e - max e) as 2^-40 fixed-point
//           integers (exact, order-independent sums); a 1024-bin histogram of
//           the masses over (max e - e) in 1/32-logit bins, then 1024 sub-bins
//           of the cut bin, isolate the few entries around the cut, which are
//           ordered by (e desc, start asc); kept = every entry at or before the
//           cut.  The children of the kept non-leaf nodes, in rank order, are
//           written as the next step's candidates; kept leaves are appended to
//           the head's attend list;
//   attend  (all CTAs) every head's attended keys (kept blocks, sink, tail)
//           are cut into chunks; CTAs own contiguous ranges of chunks, warps
//           run an online softmax per chunk, and each CTA merges its chunks per
//           head into one partial;
//   combine (one CTA per head) the partials of each head -> O.
#include "zha_args.cuh"

namespace zha {

struct Entry {
  uint32_t key;   // desc_key(e)
  uint32_t code;  // node_code(level, index)
};

constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kUnionBytes = 200 * 1024;            // select cache / score rings / attend partials
constexpr int kCache8 = kUnionBytes / 8;           // entries cached with their codes
constexpr int kCache4 = kUnionBytes / 4;           // entries cached as keys only
constexpr int kBins = 1024;
constexpr float kBinScale = 32.f;
constexpr int kMaxHeads = 1024;                    // sequences x query heads per call
constexpr int kItemsPerCta = 256;                  // attend chunks a CTA owns at most (plus one per head)
constexpr int kMaxDecodeGrid = 256;                // CTAs per decode launch the scratch is laid out for
constexpr int kPartSlots = kUnionBytes / ((2 + 128) * 4);  // attend partials a CTA can hold
constexpr int kMaxSlots = 8;                       // score ring slots per warp
static_assert(kPartSlots >= kItemsPerCta + 32, "attend partial area too small");

struct HeadState {  // per (sequence, query head), written by the head's select CTA
  long long n_cand;   // candidates of the next step
  long long n_leaf;   // kept level-1 blocks so far
  long long scored;   // nodes scored so far
  int steps;
  int leaf0;          // leaf block 0 kept (token 0 already attended)
  long long pad[4];
};

struct __align__(16) DecSmem {
  unsigned char u[kUnionBytes];
  unsigned long long hist[kBins];
  unsigned int cnt[kBins];                  // entries per coarse bin
  long long pref[kMaxHeads + 1];            // per-head prefix of work items
  unsigned long long cut_key[32];
  unsigned long long cut_w[32];
  unsigned long long red64[kDecWarps];
  uint32_t red32[kDecWarps * 2];
  unsigned long long bcast64[4];
  int bcast32[8];
  int fail;
};

// The step's entries of one head: cached in shared memory with their codes,
// cached as keys only, or read from the global step buffer.  Three concrete
// types (no run-time switch) so that every access compiles to one load from
// the right memory.
struct ViewSmemEntries {
  const Entry* ce;
  __device__ __forceinline__ uint32_t key(int64_t i) const { return ce[i].key; }
  __device__ __forceinline__ uint32_t code(int64_t i) const { return ce[i].code; }
};
struct ViewSmemKeys {
  const uint32_t* ck;
  const Entry* g;
  __device__ __forceinline__ uint32_t key(int64_t i) const { return ck[i]; }
  __device__ __forceinline__ uint32_t code(int64_t i) const {
    return __ldcg(reinterpret_cast<const unsigned int*>(g + i) + 1);
  }
};
struct ViewGlobal {
  const Entry* g;
  __device__ __forceinline__ uint32_t key(int64_t i) const { return __ldcg(reinterpret_cast<const unsigned int*>(g + i)); }
  __device__ __forceinline__ uint32_t code(int64_t i) const {
    return __ldcg(reinterpret_cast<const unsigned int*>(g + i) + 1);
  }
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

// Distance of an entry below the maximum estimate, in fp32: x = m - e >= 0.
// Bins over x are monotone in e (fp32 subtraction and power-of-two scaling
// round monotonically), so every entry of a lower bin precedes every entry of
// a higher bin in the (e desc, start asc) order, and equal estimates share a
// bin.  Coarse bins are 1/32 logit wide (kBins of them, the last one open);
// fine bins split a coarse bin into kBins parts of 1/32768 logit.
__device__ __forceinline__ float entry_gap(float m, uint32_t key) { return __fsub_rn(m, desc_key_value(key)); }
__device__ __forceinline__ int coarse_bin(float x) { return int(fminf(__fmul_rn(x, kBinScale), float(kBins - 1))); }
__device__ __forceinline__ int fine_bin(float x, int cb) {
  const float y = fminf(__fmul_rn(x, kBinScale * float(kBins)), float(kBins) * float(kBins) - 1.f);
  return min(int(y) - cb * kBins, kBins - 1);
}

__device__ __forceinline__ unsigned long long entry_mass(float m, uint32_t key) {
  const float w = expf(__fsub_rn(desc_key_value(key), m));
  return __float2ull_rn(w * 1099511627776.0f);  // 2^40
}

// Phase timestamp (profiling builds pass a buffer of 128 slots per CTA).
__device__ __forceinline__ void stamp(const DecodeArgs& a, int slot) {
  if (a.phase_ns != nullptr && threadIdx.x == 0 && slot < 128) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    a.phase_ns[blockIdx.x * 128 + slot] = t;
  }
}

// Add (count 1, mass w) to shared-memory histogram bin `bin` for every lane of
// the warp (bin < 0: nothing).  Lanes holding consecutive entries usually share
// a bin (siblings sit next to each other in a step's candidate list), so the
// lanes whose bin equals lane 0's or lane 31's are summed with the hardware
// warp reduction (the 40-bit masses split into 20-bit halves so that 32 of
// them fit 32 bits) and added by one lane; the remaining lanes add their own.
// Every lane of the warp must call it.
__device__ __forceinline__ void hist_add_warp(unsigned long long* hist, unsigned int* cnt, int bin,
                                              unsigned long long w) {
  const int lane = threadIdx.x & 31;
  const int b0 = __shfl_sync(0xffffffffu, bin, 0);
  const int b1 = __shfl_sync(0xffffffffu, bin, 31);
  const bool in0 = bin == b0, in1 = !in0 && bin == b1;
  const unsigned lo = unsigned(w & 0xfffffull), hi = unsigned(w >> 20);
  const unsigned lo0 = __reduce_add_sync(0xffffffffu, in0 ? lo : 0u);
  const unsigned hi0 = __reduce_add_sync(0xffffffffu, in0 ? hi : 0u);
  const unsigned c0 = __popc(__ballot_sync(0xffffffffu, in0));
  if (lane == 0 && b0 >= 0) {
    atomicAdd(&hist[b0], (unsigned long long)lo0 + ((unsigned long long)hi0 << 20));
    if (cnt) atomicAdd(&cnt[b0], c0);
  }
  if (b1 != b0) {
    const unsigned lo1 = __reduce_add_sync(0xffffffffu, in1 ? lo : 0u);
    const unsigned hi1 = __reduce_add_sync(0xffffffffu, in1 ? hi : 0u);
    const unsigned c1 = __popc(__ballot_sync(0xffffffffu, in1));
    if (lane == 31 && b1 >= 0) {
      atomicAdd(&hist[b1], (unsigned long long)lo1 + ((unsigned long long)hi1 << 20));
      if (cnt) atomicAdd(&cnt[b1], c1);
    }
  }
  if (!in0 && !in1 && bin >= 0) {
    atomicAdd(&hist[bin], w);
    if (cnt) atomicAdd(&cnt[bin], 1u);
  }
}

// Over kBins mass bins (shared memory), find the bin where the running mass,
// starting from `base`, first reaches `target`: returns the bin and the mass
// before it (all threads).  -1 if no bin does.
__device__ __forceinline__ int find_cut_bin(DecSmem& sm, unsigned long long base, unsigned long long target,
                                            unsigned long long* below_out) {
  constexpr int BPT = kBins / kDecThreads;
  const int tid = threadIdx.x;
  unsigned long long local = 0;
#pragma unroll
  for (int k = 0; k < BPT; ++k) local += sm.hist[tid * BPT + k];
  unsigned long long total;
  unsigned long long before = base + block_scan_u64(local, sm.red64, &total);
  if (tid == 0) sm.bcast32[0] = -1;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < BPT; ++k) {
    const unsigned long long hb = sm.hist[tid * BPT + k];
    if (before < target && before + hb >= target) {
      sm.bcast32[0] = tid * BPT + k;
      sm.bcast64[0] = before;
    }
    before += hb;
  }
  __syncthreads();
  const int bin = sm.bcast32[0];
  *below_out = sm.bcast64[0];
  __syncthreads();
  return bin;
}


// The cut for at most kDecThreads entries: thread i takes entry i, counts the
// entries ordered before it (its rank), the masses are placed in rank order
// and scanned, and the cut is the first entry whose running mass reaches T.
template <class View>
__device__ __forceinline__ unsigned long long select_cut_small(const DecodeArgs& a, const View& E, int64_t n, float m,
                                               DecSmem& sm) {
  const int tid = threadIdx.x;
  unsigned long long* k64s = sm.hist;                        // [n] order keys
  unsigned long long* wr = sm.hist + kDecThreads;            // [n] masses in rank order
  unsigned long long myk = ~0ull, myw = 0;
  if (tid < n) {
    const uint32_t k = E.key(tid);
    myk = entry_key64(a, Entry{k, E.code(tid)});
    myw = entry_mass(m, k);
    k64s[tid] = myk;
  }
  __syncthreads();
  int rank = 0;
  if (tid < n) {
    for (int j = 0; j < n; ++j) rank += k64s[j] < myk;
    wr[rank] = myw;
  }
  __syncthreads();
  const unsigned long long w_sorted = tid < n ? wr[tid] : 0ull;
  unsigned long long Z;
  const unsigned long long before = block_scan_u64(w_sorted, sm.red64, &Z);
  const unsigned long long T = ceil_p_times(Z, a.p_mant, a.p_shift);
  // sorted position of the cut: the first with before + w >= T
  if (tid == 0) sm.bcast32[2] = int(n) - 1;
  __syncthreads();
  if (tid < n && before < T && before + w_sorted >= T) sm.bcast32[2] = tid;
  __syncthreads();
  const int cut_pos = sm.bcast32[2];
  if (tid < n && rank == cut_pos) sm.bcast64[1] = myk;
  __syncthreads();
  const unsigned long long cut = sm.bcast64[1];
  __syncthreads();
  return cut;
}

// The cut of one routing step: the largest 64-bit order key (e desc, start
// asc) that is kept.  Every thread returns the same value.
// Smallest key in [lo, 2^32) whose bin (a monotone non-decreasing function of
// the key over the keys that occur) is >= target; 2^32 if none.  Every thread
// computes it (32 steps), so no broadcast is needed.
template <typename BinFn>
__device__ __forceinline__ unsigned long long first_key_at_least(uint32_t lo, int target, BinFn bin) {
  unsigned long long L = lo, H = 0x100000000ull;  // answer in [L, H]
  while (L < H) {
    const unsigned long long mid = (L + H) >> 1;
    if (bin(uint32_t(mid)) >= target) H = mid; else L = mid + 1;
  }
  return L;
}

// The cut of one routing step: the largest 64-bit order key (e desc, start
// asc) that is kept.  kmin is the smallest key (largest estimate) of the step.
// Every thread returns the same value.
template <class View>
__device__ __forceinline__ unsigned long long select_cut(const DecodeArgs& a, const View& E, int64_t n, uint32_t kmin,
                                         DecSmem& sm, int step) {
  const int tid = threadIdx.x, lane = tid & 31;
  stamp(a, 64 + 8 * step);
  if (a.p_all) return ~0ull;
  const float m = desc_key_value(kmin);
  if (n <= kDecThreads) return select_cut_small(a, E, n, m, sm);

  // coarse histogram of the masses (and counts); total mass Z and the target T = ceil(p Z)
  for (int i = tid; i < kBins; i += kDecThreads) {
    sm.hist[i] = 0ull;
    sm.cnt[i] = 0u;
  }
  __syncthreads();
  const int n32 = int(n);
  const int wseg = (n32 + kDecWarps - 1) / kDecWarps;               // entries per warp, contiguous
  const int wlo = min(n32, (tid >> 5) * wseg), whi = min(n32, wlo + wseg);
  constexpr int U = 4;                                              // groups of 32 in flight per warp
  for (int base = wlo; base < whi; base += 32 * U) {
    int bin[U];
    unsigned long long w[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + 32 * u + lane;
      bin[u] = -1;
      w[u] = 0;
      if (i < whi) {
        const uint32_t k = E.key(i);
        bin[u] = coarse_bin(entry_gap(m, k));
        w[u] = entry_mass(m, k);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) hist_add_warp(sm.hist, sm.cnt, bin[u], w[u]);
  }
  __syncthreads();
  unsigned long long Z = 0;
  {
    constexpr int BPT = kBins / kDecThreads;
    unsigned long long local = 0;
#pragma unroll
    for (int k = 0; k < BPT; ++k) local += sm.hist[tid * BPT + k];
    block_scan_u64(local, sm.red64, &Z);
  }
  const unsigned long long T = ceil_p_times(Z, a.p_mant, a.p_shift);  // keep while mass before < T
  stamp(a, 65 + 8 * step);
  unsigned long long below;
  const int cb = find_cut_bin(sm, 0ull, T, &below);
  if (cb < 0) return ~0ull;  // cannot happen for 0 < p < 1; keep everything
  auto cbin = [&](uint32_t k) { return coarse_bin(entry_gap(m, k)); };
  // keys of coarse bin cb form the contiguous range [klo, khi)
  const unsigned long long klo = first_key_at_least(kmin, cb, cbin);
  const unsigned long long khi = cb + 1 < kBins ? first_key_at_least(uint32_t(klo), cb + 1, cbin) : 0x100000000ull;

  // fine histogram inside the cut coarse bin, unless that bin is small already
  const bool use_fine = sm.cnt[cb] > 32u;
  unsigned long long flo = klo, fhi = khi;  // key range of the entries around the cut
  unsigned long long below2 = below;
  if (use_fine) {
    for (int i = tid; i < kBins; i += kDecThreads) sm.hist[i] = 0ull;
    __syncthreads();
    for (int base = wlo; base < whi; base += 32 * U) {
      int bin[U];
      unsigned long long w[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + 32 * u + lane;
        bin[u] = -1;
        w[u] = 0;
        if (i < whi) {
          const uint32_t k = E.key(i);
          if (k >= klo && k < khi) {
            bin[u] = fine_bin(entry_gap(m, k), cb);
            w[u] = entry_mass(m, k);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) hist_add_warp(sm.hist, nullptr, bin[u], w[u]);
    }
    __syncthreads();
    int fb;
    fb = find_cut_bin(sm, below, T, &below2);
    if (fb < 0) return ~0ull;
    auto fbin = [&](uint32_t k) {
      const float x = entry_gap(m, k);
      return coarse_bin(x) > cb ? kBins : fine_bin(x, cb);
    };
    flo = first_key_at_least(uint32_t(klo), fb, fbin);
    fhi = fb + 1 < kBins ? first_key_at_least(uint32_t(flo), fb + 1, fbin) : khi;
    if (fhi > khi) fhi = khi;
  }
  auto in_cut = [&](uint32_t k) { return k >= flo && k < fhi; };
  stamp(a, 66 + 8 * step);

  // gather the entries around the cut
  if (tid == 0) sm.bcast32[1] = 0;
  __syncthreads();
  for (int i = tid; i < n32; i += kDecThreads) {
    const uint32_t k = E.key(i);
    if (in_cut(k)) {
      const int s = atomicAdd(&sm.bcast32[1], 1);
      if (s < 32) {
        sm.cut_key[s] = entry_key64(a, Entry{k, E.code(i)});
        sm.cut_w[s] = entry_mass(m, k);
      }
    }
  }
  __syncthreads();
  stamp(a, 67 + 8 * step);
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
      const unsigned hit = __ballot_sync(0xffffffffu, tid < cnt && below2 + c >= T);
      const int first = hit ? __ffs(hit) - 1 : cnt - 1;
      const unsigned long long cut = __shfl_sync(0xffffffffu, k, first);
      if (tid == 0) sm.bcast64[1] = cut;
    }
    __syncthreads();
    return sm.bcast64[1];
  }
  // Many entries share the cut fine bin (exact ties or near-ties): radix
  // select on the 64-bit order key, 8 bits per pass, over that bin's entries.
  unsigned long long prefix = 0, acc_below = below2;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = tid; i < 256; i += kDecThreads) sm.hist[i] = 0ull;
    __syncthreads();
    for (int64_t i = tid; i < n; i += kDecThreads) {
      const uint32_t k = E.key(i);
      if (!in_cut(k)) continue;
      const unsigned long long k64 = entry_key64(a, Entry{k, E.code(i)});
      if (pass > 0 && (k64 >> (shift + 8)) != (prefix >> (shift + 8))) continue;
      atomicAdd(&sm.hist[(k64 >> shift) & 255], entry_mass(m, k));
    }
    __syncthreads();
    if (tid < 32) {
      // warp-parallel search over the 256 digit bins (8 per lane)
      unsigned long long loc = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) loc += sm.hist[tid * 8 + k];
      unsigned long long c = loc;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, c, off);
        if (tid >= off) c += y;
      }
      unsigned long long before = acc_below + c - loc;
      int digit = -1;
      unsigned long long dbelow = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const unsigned long long hb = sm.hist[tid * 8 + k];
        if (digit < 0 && before < T && before + hb >= T) { digit = tid * 8 + k; dbelow = before; }
        before += hb;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, digit >= 0);
      const int src = hit ? __ffs(hit) - 1 : 31;
      const int dg = __shfl_sync(0xffffffffu, hit ? digit : 255, src);
      const unsigned long long db = __shfl_sync(0xffffffffu, dbelow, src);
      if (tid == 0) {
        sm.bcast64[2] = prefix | (uint64_t(dg) << shift);
        sm.bcast64[3] = hit ? db : acc_below;
      }
    }
    __syncthreads();
    prefix = sm.bcast64[2];
    acc_below = sm.bcast64[3];
    __syncthreads();
  }
  return prefix;
}

// Grid barrier over all CTAs of the cooperative launch: a 64-bit arrival
// counter that only grows; barrier k of a launch completes when it reaches
// base + k * gridDim.x (the host tracks the base).  Returns true for every
// thread of the CTA if the wait gave up.
__device__ __forceinline__ bool grid_sync(const DecodeArgs& a, DecSmem& sm, unsigned long long& target) {
  target += gridDim.x;
  __syncthreads();
  if (threadIdx.x == 0) {
    sm.fail = 0;
    __threadfence();
    asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(a.bar) : "memory");
    long long it = 0;
    while (true) {
      unsigned long long v;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(a.bar) : "memory");
      if (v >= target) break;
      if (++it > a.spin_limit) {
        sm.fail = 1;
        raise_status(a.t.status, ZHA_ERR_TIMEOUT);
        break;
      }
      __nanosleep(20);
    }
  }
  __syncthreads();
  return sm.fail != 0;
}

// Inclusive prefix of per-head counts held in sm.pref[1..nh] (pref[0] = 0); returns the total.
__device__ __forceinline__ long long build_prefix(DecSmem& sm, int nh) {
  long long carry = 0;
  for (int base = 0; base < nh; base += kDecThreads) {
    const int i = base + threadIdx.x;
    const unsigned long long v = i < nh ? (unsigned long long)sm.pref[1 + i] : 0ull;
    unsigned long long tot;
    const unsigned long long ex = block_scan_u64(v, sm.red64, &tot);
    if (i < nh) sm.pref[1 + i] = carry + (long long)(ex + v);
    carry += (long long)tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) sm.pref[0] = 0;
  __syncthreads();
  return carry;
}

// Head owning work item i: the largest h with pref[h] <= i.
__device__ __forceinline__ int owner_of(const DecSmem& sm, int nh, long long i) {
  int lo = 0, hi = nh - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sm.pref[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ bool valid_code(const DecodeArgs& a, uint32_t code) {
  const int l = code_level(code);
  return l >= 1 && l <= a.t.levels && int64_t(code_index(code)) < a.nl[l];
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// wait until at most `pending` of this thread's newest groups are still in flight
__device__ __forceinline__ void cp_async_wait(int pending) {
  switch (pending) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
    case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
    case 5: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
    case 6: asm volatile("cp.async.wait_group 6;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 7;" ::: "memory"); break;
  }
}

// Estimate of a node whose record sits in shared memory (whole warp; the
// lane's q slice covers elements [cl*EPC, cl*EPC+EPC), cl = lane % CPR).
template <typename T, int D>
__device__ __forceinline__ float score_record_smem(const unsigned char* rec, int R, float inv_sqrt_d,
                                                   const float* qs, int lane) {
  constexpr int EPC = 16 / sizeof(T);
  constexpr int CPR = D * sizeof(T) / 16;
  constexpr int RPI = 32 / CPR;
  const float* bias = reinterpret_cast<const float*>(rec + size_t(R) * D * sizeof(T));
  const int sub = lane / CPR, cl = lane % CPR;
  float best = -INFINITY;
  for (int j0 = 0; j0 < R; j0 += RPI) {
    const int j = j0 + sub;
    float part = 0.f;
    if (j < R) {
      const uint4 v = *reinterpret_cast<const uint4*>(rec + (size_t(j) * CPR + cl) * 16);
      float x[EPC];
      unpack16<T>(v, x);
#pragma unroll
      for (int i = 0; i < EPC; ++i) part = fmaf(x[i], qs[i], part);
    }
#pragma unroll
    for (int off = CPR / 2; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (j < R) best = fmaxf(best, fmaf(part, inv_sqrt_d, bias[j]));
  }
#pragma unroll
  for (int off = 16; off >= CPR; off >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, off));
  return best;
}

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(DecodeArgs a) {
  constexpr int EPC = 16 / sizeof(T);
  constexpr int CPR = D * sizeof(T) / 16;
  constexpr int KPW = 32 / CPR;  // keys per warp pass in the attention loop
  extern __shared__ __align__(16) unsigned char smem_raw[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nh = a.nheads;
  const int b = a.t.block;
  const int R = a.t.refs;
  const long long gwarp = (long long)blockIdx.x * kDecWarps + wid;
  const long long nwarps = (long long)gridDim.x * kDecWarps;
  unsigned long long bar_target = a.bar_base;
  auto ws = [&](int h) { return a.ws + uint64_t(h) * a.ws_per_bh; };
  auto sel = [&](int h) { return reinterpret_cast<Entry*>(ws(h)); };
  auto cand = [&](int h) { return reinterpret_cast<uint32_t*>(ws(h) + a.cap_sel * sizeof(Entry)); };
  auto leaves = [&](int h) { return reinterpret_cast<uint32_t*>(ws(h) + a.cap_sel * (sizeof(Entry) + 4)); };
  auto hstate = [&](int h) {
    return reinterpret_cast<HeadState*>(ws(h) + a.cap_sel * (sizeof(Entry) + 4) + a.cap_list * 4);
  };
  auto q_slice = [&](int h, float* qs) {
    const T* q = static_cast<const T*>(a.Q) + size_t(h) * D + (lane % CPR) * EPC;
    unpack16<T>(*reinterpret_cast<const uint4*>(q), qs);
  };
  const int rec_bytes = int(a.t.rec_bytes);
  const int rec_chunks = rec_bytes / 16;
  const int nslot = max(1, min(kMaxSlots, (kUnionBytes / kDecWarps) / rec_bytes));
  unsigned char* ring = sm.u + size_t(wid) * nslot * rec_bytes;

  stamp(a, 0);
  for (int step = 0; step < a.n_steps; ++step) {
    // ---------------- score (all CTAs)
    for (int i = tid; i < nh; i += kDecThreads) {
      long long c = a.n_roots;
      if (step > 0) c = min64(max64(__ldcg(&hstate(i)->n_cand), 0), a.cap_sel);
      sm.pref[1 + i] = c;
    }
    __syncthreads();
    const long long total = build_prefix(sm, nh);
    {
      const long long i0 = gwarp * total / nwarps, i1 = (gwarp + 1) * total / nwarps;
      const long long cnt = i1 - i0;
      // codes of the next 32 items, one per lane
      uint32_t code_reg = 0;
      int head_reg = 0;
      auto fetch_codes = [&](long long k0) {
        const long long it = i0 + k0 + lane;
        code_reg = 0;
        head_reg = 0;
        if (k0 + lane < cnt) {
          const int h = owner_of(sm, nh, it);
          const long long pos = it - sm.pref[h];
          uint32_t code = step == 0 ? root_code(a, pos) : __ldcg(cand(h) + pos);
          if (!valid_code(a, code)) {
            raise_status(a.t.status, ZHA_ERR_CAPACITY);
            code = 0;  // marks an item to skip
          }
          code_reg = code;
          head_reg = h;
        }
      };
      long long issued = 0, done = 0;
      int qhead = -1;
      float qs[EPC];
      if (cnt > 0) fetch_codes(0);
      while (done < cnt) {
        // keep up to nslot records in flight
        while (issued < cnt && issued - done < nslot && (issued >> 5) == (done >> 5)) {
          const uint32_t code = __shfl_sync(0xffffffffu, code_reg, int(issued & 31));
          const int h = __shfl_sync(0xffffffffu, head_reg, int(issued & 31));
          unsigned char* slot = ring + size_t(issued % nslot) * rec_bytes;
          if (code != 0) {
            const int kvh = (h % a.t.hq) / a.t.group;
            const unsigned char* src =
                reinterpret_cast<const unsigned char*>(a.t.rec(code_level(code), kvh, code_index(code)));
            for (int c = lane; c < rec_chunks; c += 32) cp_async16(slot + c * 16, src + c * 16);
          }
          cp_async_commit();
          ++issued;
        }
        const uint32_t code = __shfl_sync(0xffffffffu, code_reg, int(done & 31));
        const int h = __shfl_sync(0xffffffffu, head_reg, int(done & 31));
        if (code != 0 && h != qhead) {  // load the head's query while the record is in flight
          q_slice(h, qs);
          qhead = h;
        }
        cp_async_wait(int(issued - done - 1));
        __syncwarp();
        if (code != 0) {
          const float e = score_record_smem<T, D>(ring + size_t(done % nslot) * rec_bytes, R, a.t.inv_sqrt_d, qs,
                                                  lane);
          if (lane == 0) sel(h)[i0 + done - sm.pref[h]] = Entry{desc_key(e), code};
        }
        __syncwarp();
        ++done;
        if ((done & 31) == 0 && done < cnt) fetch_codes(done);
      }
    }
    stamp(a, 1 + 4 * step);
    if (grid_sync(a, sm, bar_target)) return;
    stamp(a, 2 + 4 * step);

    // ---------------- select (one CTA per head)
    for (int h = blockIdx.x; h < nh; h += gridDim.x) {
      const long long n = sm.pref[h + 1] - sm.pref[h];
      HeadState* hs = hstate(h);
      long long n_leaf0 = 0, scored0 = 0;
      int leaf0 = 0, steps0 = 0;
      if (step > 0) {
        n_leaf0 = min64(max64(__ldcg(&hs->n_leaf), 0), a.cap_list);
        scored0 = __ldcg(&hs->scored);
        leaf0 = __ldcg(&hs->leaf0);
        steps0 = __ldcg(&hs->steps);
      }
      if (n == 0) {
        if (tid == 0) {
          hs->n_cand = 0;
          hs->n_leaf = n_leaf0;
          hs->scored = scored0;
          hs->leaf0 = leaf0;
          hs->steps = steps0;
        }
        continue;
      }
      const Entry* S = sel(h);
      const int mode = n <= kCache8 ? 1 : (n <= kCache4 ? 2 : 0);
      __syncthreads();
      uint32_t kmin = 0xffffffffu;
      if (mode == 1) {
        Entry* ce = reinterpret_cast<Entry*>(sm.u);
        for (long long i = tid; i < n; i += kDecThreads) {
          const uint2 v = __ldcg(reinterpret_cast<const uint2*>(S + i));
          ce[i] = Entry{v.x, v.y};
          kmin = min(kmin, v.x);
        }
      } else if (mode == 2) {
        uint32_t* ck = reinterpret_cast<uint32_t*>(sm.u);
        for (long long i = tid; i < n; i += kDecThreads) {
          const uint32_t k = __ldcg(reinterpret_cast<const unsigned int*>(S + i));
          ck[i] = k;
          kmin = min(kmin, k);
        }
      } else {
        for (long long i = tid; i < n; i += kDecThreads)
          kmin = min(kmin, __ldcg(reinterpret_cast<const unsigned int*>(S + i)));
      }
      kmin = block_min_u32(kmin, sm.red32);  // includes the barrier that publishes the cache
      int my_leaf0 = 0;
      uint32_t tot_leaf = 0, tot_par = 0;
      auto select_and_rank = [&](const auto& E) {
      if (a.scored) {
        int32_t* out = a.scored + size_t(h) * a.scored_cap;
        for (long long i = tid; i < n; i += kDecThreads)
          if (scored0 + i < a.scored_cap) out[scored0 + i] = int32_t(E.code(i));
      }
      stamp(a, 32 + 3 * step);
      const unsigned long long cut = select_cut(a, E, n, kmin, sm, step);
      stamp(a, 33 + 3 * step);
      const uint32_t cut32 = uint32_t(cut >> 32);
      // ranks of the kept entries in canonical order: each warp owns a contiguous
      // segment, walked 32 entries at a time (coalesced reads and writes)
      const int64_t wseg = (n + kDecWarps - 1) / kDecWarps;
      const int64_t wlo = min64(n, wid * wseg), whi = min64(n, wlo + wseg);
      auto kept_entry = [&](long long i, uint32_t& code) {
        const uint32_t k = E.key(i);
        if (k > cut32) return false;
        code = E.code(i);
        return k < cut32 || entry_key64(a, Entry{k, code}) <= cut;
      };
      uint32_t wleaf = 0, wpar = 0;
      for (int64_t base = wlo; base < whi; base += 128) {
        bool kp[4];
        uint32_t code[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t i = base + 32 * u + lane;
          code[u] = 0;
          kp[u] = i < whi && kept_entry(i, code[u]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          wleaf += __popc(__ballot_sync(0xffffffffu, kp[u] && code_level(code[u]) == 1));
          wpar += __popc(__ballot_sync(0xffffffffu, kp[u] && code_level(code[u]) != 1));
        }
      }
      if (lane == 0) {
        sm.red32[wid] = wleaf;
        sm.red32[kDecWarps + wid] = wpar;
      }
      __syncthreads();
      stamp(a, 68 + 8 * step);
      uint32_t leaf_off = 0, par_off = 0;
      for (int w = 0; w < kDecWarps; ++w) {
        const uint32_t l = sm.red32[w], q = sm.red32[kDecWarps + w];
        if (w < wid) { leaf_off += l; par_off += q; }
        tot_leaf += l;
        tot_par += q;
      }
      const unsigned below_me = (1u << lane) - 1u;
      for (int64_t base = wlo; base < whi; base += 32) {
        const int64_t i = base + lane;
        uint32_t code = 0;
        const bool kp = i < whi && kept_entry(i, code);
        const bool isleaf = kp && code_level(code) == 1;
        const bool ispar = kp && code_level(code) != 1;
        const unsigned ml = __ballot_sync(0xffffffffu, isleaf);
        const unsigned mp = __ballot_sync(0xffffffffu, ispar);
        if (isleaf) {
          const long long g = n_leaf0 + leaf_off + __popc(ml & below_me);
          if (code_index(code) == 0) my_leaf0 = 1;
          if (g < a.cap_list) leaves(h)[g] = code_index(code);
          else raise_status(a.t.status, ZHA_ERR_CAPACITY);
          if (a.kept && g < a.kept_stride) a.kept[size_t(h) * a.kept_stride + g] = int32_t(code_index(code));
        }
        if (ispar) {
          const long long pr = par_off + __popc(mp & below_me);
          const uint32_t cl = code_level(code) - 1, ci = code_index(code) * uint32_t(b);
          if ((pr + 1) * b <= a.cap_sel) {
            for (int c = 0; c < b; ++c) cand(h)[pr * b + c] = node_code(cl, ci + uint32_t(c));
          }
        }
        leaf_off += __popc(ml);
        par_off += __popc(mp);
      }
      };
      if (mode == 1) select_and_rank(ViewSmemEntries{reinterpret_cast<const Entry*>(sm.u)});
      else if (mode == 2) select_and_rank(ViewSmemKeys{reinterpret_cast<const uint32_t*>(sm.u), S});
      else select_and_rank(ViewGlobal{S});
      my_leaf0 = __syncthreads_or(my_leaf0);
      stamp(a, 69 + 8 * step);
      if (tid == 0) {
        long long nc = (long long)tot_par * b;
        if (nc > a.cap_sel) {
          raise_status(a.t.status, ZHA_ERR_CAPACITY);
          nc = 0;
        }
        hs->n_cand = nc;
        hs->n_leaf = min64(n_leaf0 + tot_leaf, a.cap_list);
        hs->scored = scored0 + n;
        hs->leaf0 = leaf0 | my_leaf0;
        hs->steps = steps0 + 1;
      }
      __syncthreads();
    }
    stamp(a, 3 + 4 * step);
    if (grid_sync(a, sm, bar_target)) return;
    stamp(a, 4 + 4 * step);
  }

  // ---------------- attend (all CTAs)
  const long long n1 = a.nl[1];
  const long long tail = a.n_tokens - n1 * b;
  auto head_keys = [&](int h, long long& nl, bool& sink) {
    nl = 0;
    int l0 = 0;
    if (a.n_steps > 0) {
      nl = min64(max64(__ldcg(&hstate(h)->n_leaf), 0), a.cap_list);
      l0 = __ldcg(&hstate(h)->leaf0);
    }
    sink = (n1 > 0) && !l0;
    return nl * b + (sink ? 1 : 0) + tail;
  };
  for (int i = tid; i < nh; i += kDecThreads) {
    long long nl;
    bool sink;
    sm.pref[1 + i] = head_keys(i, nl, sink);
  }
  __syncthreads();
  const long long total_keys = build_prefix(sm, nh);
  // chunk size: at least 32 keys, large enough that a CTA owns <= kItemsPerCta chunks (+1 per head)
  long long chunk = (total_keys + (long long)gridDim.x * kItemsPerCta - 1) / ((long long)gridDim.x * kItemsPerCta);
  chunk = max64(32, chunk);
  for (int i = tid; i < nh; i += kDecThreads) {
    long long nl;
    bool sink;
    sm.pref[1 + i] = (head_keys(i, nl, sink) + chunk - 1) / chunk;
  }
  __syncthreads();
  const long long total_items = build_prefix(sm, nh);
  stamp(a, 60);
  const long long c0 = (long long)blockIdx.x * total_items / gridDim.x;
  const long long c1 = min64((long long)(blockIdx.x + 1) * total_items / gridDim.x, c0 + kPartSlots);
  if (tid == 0 && (long long)(blockIdx.x + 1) * total_items / gridDim.x > c1) raise_status(a.t.status, ZHA_ERR_CAPACITY);
  float (*part)[2 + 128] = reinterpret_cast<float (*)[2 + 128]>(sm.u);
  {
    const int sub = lane / CPR, cl = lane % CPR;
    constexpr int kU = 8;
    for (long long it = c0 + wid; it < c1; it += kDecWarps) {
      const int h = owner_of(sm, nh, it);
      const long long ci = it - sm.pref[h];
      const int kvh = (h % a.t.hq) / a.t.group;
      long long nl;
      bool sink;
      const long long kh = head_keys(h, nl, sink);
      const long long leaf_keys = nl * b;
      const long long k0 = ci * chunk, k1 = min64(kh, k0 + chunk);
      float qs[EPC];
      q_slice(h, qs);
      const T* Kh = static_cast<const T*>(a.t.K) + size_t(kvh) * a.t.capacity * D;
      const T* Vh = static_cast<const T*>(a.t.V) + size_t(kvh) * a.t.capacity * D;
      const uint32_t* lv = leaves(h);
      // leaf indices of the chunk's first 32 blocks, one per lane
      const long long lf0 = k0 / b;
      uint32_t leaf_reg = 0;
      if (lf0 + lane < nl) leaf_reg = __ldcg(lv + lf0 + lane);
      float m_run = -INFINITY, l_run = 0.f, o[EPC];
#pragma unroll
      for (int i = 0; i < EPC; ++i) o[i] = 0.f;
      for (long long wb = k0; wb < k1; wb += (long long)KPW * kU) {
        uint4 kv[kU], vv[kU];
        bool ok[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const long long idx = wb + (long long)u * KPW + sub;
          ok[u] = idx < k1;
          long long tok = 0;
          const long long li = idx / b;
          // every lane takes part in the shuffle; only leaf keys use the value
          const uint32_t lr = __shfl_sync(0xffffffffu, leaf_reg, int((li - lf0) & 31));
          if (idx < leaf_keys) {
            const uint32_t leaf = (li - lf0 < 32) ? lr : __ldcg(lv + li);
            tok = int64_t(leaf) * b + idx % b;
          } else if (sink && idx == leaf_keys) {
            tok = 0;
          } else {
            tok = n1 * b + (idx - leaf_keys - (sink ? 1 : 0));
          }
          if (ok[u] && (tok < 0 || tok >= a.n_tokens)) {  // a corrupted leaf index: skip it
            ok[u] = false;
            raise_status(a.t.status, ZHA_ERR_CAPACITY);
          }
          if (ok[u]) {
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
      // merge the KPW lane groups of the warp (lanes l, l+CPR, ... hold the same d-range)
#pragma unroll
      for (int off = CPR; off < 32; off <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m_run, off);
        const float lo2 = __shfl_xor_sync(0xffffffffu, l_run, off);
        const float mn = fmaxf(m_run, mo);
        const float sa = m_run == -INFINITY ? 0.f : expf(m_run - mn);
        const float sb = mo == -INFINITY ? 0.f : expf(mo - mn);
#pragma unroll
        for (int i = 0; i < EPC; ++i) {
          const float oo = __shfl_xor_sync(0xffffffffu, o[i], off);
          o[i] = o[i] * sa + oo * sb;
        }
        l_run = l_run * sa + lo2 * sb;
        m_run = mn;
      }
      float* P = part[it - c0];
      if (lane == 0) {
        P[0] = m_run;
        P[1] = l_run;
      }
      if (lane < CPR) {
#pragma unroll
        for (int i = 0; i < EPC; ++i) P[2 + cl * EPC + i] = o[i];
      }
    }
  }
  __syncthreads();
  stamp(a, 26);
  // merge this CTA's chunks per head segment; one partial per segment, stored at
  // the global slot of the segment's first chunk
  for (long long seg = c0 + wid; seg < c1; seg += kDecWarps) {
    const int h = owner_of(sm, nh, seg);
    if (seg != c0 && seg != sm.pref[h]) continue;  // not the first chunk of a segment
    const long long send = min64(c1, sm.pref[h + 1]);
    float M = -INFINITY;
    for (long long j = seg; j < send; ++j) M = fmaxf(M, part[j - c0][0]);
    float L = 0.f;
    float acc[(D + 31) / 32];
#pragma unroll
    for (int q = 0; q < (D + 31) / 32; ++q) acc[q] = 0.f;
    for (long long j = seg; j < send; ++j) {
      const float mj = part[j - c0][0];
      if (mj == -INFINITY) continue;
      const float sc = expf(mj - M);
      L = fmaf(sc, part[j - c0][1], L);
#pragma unroll
      for (int q = 0; q < (D + 31) / 32; ++q)
        if (q * 32 + lane < D) acc[q] = fmaf(sc, part[j - c0][2 + q * 32 + lane], acc[q]);
    }
    float* G = a.attn_part + size_t(seg) * (2 + D);
    if (lane == 0) {
      G[0] = M;
      G[1] = L;
    }
#pragma unroll
    for (int q = 0; q < (D + 31) / 32; ++q)
      if (q * 32 + lane < D) G[2 + q * 32 + lane] = acc[q];
  }
  stamp(a, 27);
  if (grid_sync(a, sm, bar_target)) return;
  stamp(a, 28);

  // ---------------- combine (one CTA per head)
  for (int h = blockIdx.x; h < nh; h += gridDim.x) {
    const long long p0 = sm.pref[h], p1 = sm.pref[h + 1];
    // partial slots: one per CTA whose chunk range meets [p0, p1), at max(p0, range start)
    float M = -INFINITY;
    auto range_start = [&](long long c) { return (c * total_items) / (long long)gridDim.x; };
    long long cfirst = (p0 * gridDim.x) / max64(total_items, 1);
    while (cfirst > 0 && range_start(cfirst) > p0) --cfirst;
    while (cfirst + 1 < gridDim.x && range_start(cfirst + 1) <= p0) ++cfirst;
    for (long long c = cfirst + tid; c < gridDim.x; c += kDecThreads) {
      const long long cs = max64(p0, range_start(c));
      if (cs >= p1) break;
      if (cs >= min64(p1, range_start(c + 1))) continue;  // empty range
      M = fmaxf(M, __ldcg(a.attn_part + size_t(cs) * (2 + D)));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (lane == 0) sm.red32[wid] = __float_as_uint(M);
    __syncthreads();
    M = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, __uint_as_float(sm.red32[w]));
    __syncthreads();
    float L = 0.f, acc = 0.f;
    const int e = tid % D, prt = tid / D;  // NP threads per output element
    constexpr int NP = kDecThreads / D;
    float Lp = 0.f;
    for (long long c = cfirst + prt; c < gridDim.x; c += NP) {
      const long long cs = max64(p0, range_start(c));
      if (cs >= p1) break;
      if (cs >= min64(p1, range_start(c + 1))) continue;  // empty range
      const float* G = a.attn_part + size_t(cs) * (2 + D);
      const float mg = __ldcg(G), lg = __ldcg(G + 1), og = __ldcg(G + 2 + e);  // independent loads
      const float sc = mg == -INFINITY ? 0.f : expf(mg - M);
      Lp = fmaf(sc, lg, Lp);
      acc = fmaf(sc, og, acc);
    }
    float* red = reinterpret_cast<float*>(sm.hist);  // [NP][D] + [NP]
    red[prt * D + e] = acc;
    if (e == 0) red[NP * D + prt] = Lp;
    __syncthreads();
    if (prt == 0) {
      for (int q = 1; q < NP; ++q) acc += red[q * D + e];
      for (int q = 0; q < NP; ++q) L += red[NP * D + q];
      a.O[size_t(h) * D + e] = acc / L;
    }
    if (tid == 0) {
      long long nl = 0, scored = 0;
      int l0 = 0, steps = 0;
      if (a.n_steps > 0) {
        nl = __ldcg(&hstate(h)->n_leaf);
        l0 = __ldcg(&hstate(h)->leaf0);
        scored = __ldcg(&hstate(h)->scored);
        steps = __ldcg(&hstate(h)->steps);
      }
      if (a.kept_cnt) a.kept_cnt[h] = int32_t(nl);
      if (a.stats) {
        int64_t* st = a.stats + size_t(h) * ZHA_STAT_COUNT;
        st[ZHA_STAT_NODES_SCORED] = scored;
        st[ZHA_STAT_LEAVES_KEPT] = nl;
        st[ZHA_STAT_KEYS] = nl * b + ((n1 > 0 && !l0) ? 1 : 0) + tail;
        st[ZHA_STAT_STEPS] = steps;
      }
    }
    __syncthreads();
  }
  stamp(a, 29);
}

// ------------------------------------------------------------------ host launcher
template <typename T, int D>
static int grid_size_t() {
  static int cached = -1;
  if (cached >= 0) return cached;
  auto kern = decode_kernel<T, D>;
  const size_t smem = sizeof(DecSmem);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess) return 0;
  int per_sm = 0, dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecThreads, smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cached = min(per_sm * sms, kMaxDecodeGrid);
  return cached;
}

template <typename T, int D>
static cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t st) {
  auto kern = decode_kernel<T, D>;
  const int grid = grid_size_t<T, D>();
  if (grid < 1) return cudaErrorLaunchOutOfResources;
  DecodeArgs args = a;
  void* params[] = {&args};
  count_launches(1);
  return cudaLaunchCooperativeKernel((const void*)kern, dim3(unsigned(grid)), dim3(kDecThreads), params,
                                     sizeof(DecSmem), st);
}

cudaError_t launch_decode(const DecodeArgs& a, int dtype, cudaStream_t st) {
  if (dtype == ZHA_BF16)
    return a.t.d == 128 ? launch_decode_t<__nv_bfloat16, 128>(a, st) : launch_decode_t<__nv_bfloat16, 64>(a, st);
  return a.t.d == 128 ? launch_decode_t<float, 128>(a, st) : launch_decode_t<float, 64>(a, st);
}

int decode_grid(int dtype, int d) {
  if (dtype == ZHA_BF16) return d == 128 ? grid_size_t<__nv_bfloat16, 128>() : grid_size_t<__nv_bfloat16, 64>();
  return d == 128 ? grid_size_t<float, 128>() : grid_size_t<float, 64>();
}

size_t decode_smem_bytes() { return sizeof(DecSmem); }
size_t decode_head_state_bytes() { return sizeof(HeadState); }
int decode_max_heads() { return kMaxHeads; }
int decode_items_per_cta() { return kItemsPerCta; }
int decode_max_grid() { return kMaxDecodeGrid; }

}  // namespace zha
