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
// GPU design.  A decode call is a fixed sequence of kernels on the caller's
// stream, each launched with programmatic stream serialization (it may start
// while the one before drains and waits for it before reading its output);
// all query heads of all sequences are routed together so that the whole GPU
// shares the work of the heads whose routing is diffuse.  Per routing step s:
//   score   (one CTA per SM) the step's records of every head (the roots, or
//           the b children of each kept non-leaf of step s-1) form one list
//           cut into contiguous per-warp ranges; each warp fetches its node
//           records with bulk copies into a ring of shared-memory slots, computes the estimates (tensor cores for
//           bf16) and writes (descending key of e, node code) at the entry's
//           position in its head's step buffer, adding the entry's
//           fixed-point mass to the step's histogram anchored at the largest
//           estimate of step s-1;
//   select  (one CTA per head) the cut: masses as 2^-40 fixed-point integers
//           (exact, order-independent sums); the cut bin from the anchored
//           histogram (or histograms built in the CTA), then its sub-bins,
//           isolate the few entries around the cut, which are ordered by
//           (e desc, start asc); kept = every entry at or before the cut.
//           Kept non-leaves become the next step's units, kept leaves are
//           appended to the head's attend list.
// Then
//   attend  (two CTAs per SM) every head's attended keys (kept blocks, sink,
//           tail) are cut into chunks; CTAs own contiguous ranges of chunks,
//           warps run an online softmax per chunk (tensor cores for bf16), and
//           each CTA merges its chunks per head into one partial;
//   combine (one CTA per head) the head's partials merged in a fixed order
//           -> O, the head's kept count and statistics.
// The only waits inside a kernel are a scoring warp's waits for its own bulk
// copies; they are bounded (on running out the kernel raises ZHA_ERR_TIMEOUT).
#include <cstddef>
#include <mutex>
#include <type_traits>

#include "zha_args.cuh"

namespace zha {

struct Entry {
  uint32_t key;   // desc_key(e)
  uint32_t code;  // node_code(level, index)
};

constexpr int kDecThreads = 512;                   // threads of a scoring or select CTA
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kUnionBytes = 208 * 1024;            // select: step keys and codes cached in shared memory
constexpr int kCacheEnt = kUnionBytes / 8;          // entries (key + code) the cache holds
constexpr int kSpecEnt = 512;                       // entries a select fetches before it knows the step's size
constexpr int kRingBytes = 200 * 1024;             // scoring: record ring of the CTA's warps
constexpr int kBins = 1024;
constexpr float kBinScale = 32.f;
constexpr int kMaxHeads = 1024;                    // sequences x query heads per call
constexpr int kMaxSlots = 8;                       // score ring slots per warp
constexpr long long kDrainLimit = 1ll << 30;       // bound of the wait for copies in flight after a timeout
constexpr int kAttThreads = 256;                   // threads of an attention CTA
constexpr int kAttWarps = kAttThreads / 32;
constexpr int kAttItems = 32;                      // attend chunks a CTA owns at most
constexpr int kMaxAttGrid = 512;                   // attention CTAs the scratch is laid out for

struct HeadState {  // per (sequence, query head)
  long long n[2];          // entries of the step built in each parity buffer (step 0: unused)
  long long units;         // kept non-leaves of the last select (units of the next scoring phase)
  long long scored;        // nodes scored so far
  long long n_leaf;        // kept level-1 blocks listed so far
  unsigned int kinv[2];    // ~(smallest key) of the step built in each parity buffer
  int ovf[2];              // an estimate of that step lies above its anchor span
  float anchor;            // histogram anchor of the step being built (max e of the step before)
  int steps;               // selects done
  int leaf0;               // leaf block 0 kept (token 0 already attended)
  int reserved[33];
  long long pad[7];
};
static_assert(sizeof(HeadState) == 256, "HeadState layout");

// Per-head routing state and leaf bitmaps live in one scratch region.  The
// first select of a decode starts the head's counters from zero, the last
// one leaves both parities' step extremes cleared and the export clears the
// bitmap, so a decode leaves the region ready for the next one (after an
// error status the host zeroes it).

// 32-bit words of a head's leaf bitmap (one bit per level-1 block), a multiple of 4.
__host__ __device__ __forceinline__ int64_t decode_bitmap_words(int64_t cap_sel) {
  return (((cap_sel + 31) / 32) + 3) & ~int64_t(3);
}

struct __align__(16) DecSmem {
  unsigned char u[kUnionBytes];
  unsigned long long hist[kBins];
  unsigned long long cut_key[32];
  unsigned long long cut_w[32];
  unsigned long long red64[kDecWarps];
  uint32_t red32[kDecWarps * 2];
  unsigned long long bcast64[4];
  int bcast32[8];
  DecodeArgs args;  // the kernel arguments, staged (stage_args); last, so that the arrays above keep
                    // their 16-byte alignment (the argument block is 8 mod 16 bytes long)
};
static_assert(offsetof(DecSmem, u) % 16 == 0 && offsetof(DecSmem, hist) % 16 == 0, "16-byte shared accesses");

// Division of 32-bit values by a fixed divisor d >= 2 with a multiply-high and
// one correction step (m = floor(2^32 / d) underestimates x / d by less than 1).
struct DivU32 {
  uint32_t d, m;
  __device__ explicit DivU32(uint32_t div) : d(div), m(uint32_t((1ull << 32) / div)) {}
  __device__ __forceinline__ uint32_t div(uint32_t x, uint32_t* rem) const {
    uint32_t q = __umulhi(x, m);
    uint32_t r = x - q * d;
    if (r >= d) {
      ++q;
      r -= d;
    }
    *rem = r;
    return q;
  }
};

// The step's entries of one head: keys [0, nc) cached in shared memory, the
// rest (and every code) read from the global step buffers.
struct StepView {
  const uint32_t* ck;  // cached keys
  const uint32_t* cc;  // cached codes
  int nc;              // entries cached
  const uint32_t* gk;  // global keys
  const uint32_t* gc;  // global codes
  __device__ __forceinline__ uint32_t key(int64_t i) const { return i < nc ? ck[i] : __ldcg(gk + i); }
  __device__ __forceinline__ uint32_t code(int64_t i) const { return i < nc ? cc[i] : __ldcg(gc + i); }
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

// Block-wide exclusive scan of one value per thread; returns the exclusive
// prefix and writes the block total to *total (all threads).
template <int NW = kDecWarps>
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
  // the warp totals, scanned across lanes (NW <= 32)
  unsigned long long t = lane < NW ? red[lane] : 0ull;
#pragma unroll
  for (int off = 1; off < NW; off <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, t, off);
    if (lane >= off) t += y;
  }
  const unsigned long long base = __shfl_sync(0xffffffffu, t, (wid + 31) & 31);
  *total = __shfl_sync(0xffffffffu, t, NW - 1);
  __syncthreads();
  return (wid > 0 ? base : 0ull) + x - v;
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

// Shared-memory atomics addressed in the shared window.  The select code
// reaches its shared arrays through references, which the compiler treats as
// generic addresses; a generic 64-bit atomic that collides takes a very slow
// path, so the shared-space forms are issued explicitly.
__device__ __forceinline__ void smem_add_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.shared.add.u64 [%0], %1;" ::"r"(unsigned(__cvta_generic_to_shared(p))), "l"(v) : "memory");
}
__device__ __forceinline__ int smem_inc(int* p) {
  int r;
  asm volatile("atom.shared.add.u32 %0, [%1], 1;" : "=r"(r) : "r"(unsigned(__cvta_generic_to_shared(p))) : "memory");
  return r;
}
__device__ __forceinline__ void smem_max_s32(int* p, int v) {
  asm volatile("red.shared.max.s32 [%0], %1;" ::"r"(unsigned(__cvta_generic_to_shared(p))), "r"(v) : "memory");
}

// Add mass w to shared-memory histogram bin `bin` for every lane of
// the warp (bin < 0: nothing).  Lanes holding consecutive entries usually share
// a bin (siblings sit next to each other in a step's candidate list), so the
// lanes whose bin equals lane 0's or lane 31's are summed with the hardware
// warp reduction (the 40-bit masses split into 20-bit halves so that 32 of
// them fit 32 bits) and added by one lane; the remaining lanes add their own.
// Every lane of the warp must call it.
__device__ __forceinline__ void hist_add_warp(unsigned long long* hist, int bin, unsigned long long w) {
  if (!__any_sync(0xffffffffu, bin >= 0)) return;
  const int lane = threadIdx.x & 31;
  const int b0 = __shfl_sync(0xffffffffu, bin, 0);
  const int b1 = __shfl_sync(0xffffffffu, bin, 31);
  const bool in0 = bin == b0, in1 = !in0 && bin == b1;
  const unsigned lo = unsigned(w & 0xfffffull), hi = unsigned(w >> 20);
  const unsigned lo0 = __reduce_add_sync(0xffffffffu, in0 ? lo : 0u);
  const unsigned hi0 = __reduce_add_sync(0xffffffffu, in0 ? hi : 0u);
  if (lane == 0 && b0 >= 0) smem_add_u64(&hist[b0], (unsigned long long)lo0 + ((unsigned long long)hi0 << 20));
  if (b1 != b0) {
    const unsigned lo1 = __reduce_add_sync(0xffffffffu, in1 ? lo : 0u);
    const unsigned hi1 = __reduce_add_sync(0xffffffffu, in1 ? hi : 0u);
    if (lane == 31 && b1 >= 0) smem_add_u64(&hist[b1], (unsigned long long)lo1 + ((unsigned long long)hi1 << 20));
  }
  if (!in0 && !in1 && bin >= 0) smem_add_u64(&hist[bin], w);
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


// The cut for at most kDecThreads entries: thread i takes entry i; the order
// keys are sorted by a bitonic network in shared memory (strides below 32
// within a warp by shuffles), the masses scanned in sorted order, and the cut
// is the first entry whose running mass reaches T.
template <class View>
__device__ __noinline__ unsigned long long select_cut_small(const DecodeArgs& a, const View E, int64_t n, float m,
                                                            DecSmem& sm, int step) {
  const int tid = threadIdx.x;
  unsigned long long* ks = sm.hist;  // [np] order keys
  int np = 32;
  while (np < n) np <<= 1;  // <= kDecThreads
  unsigned long long k = ~0ull;
  if (tid < n) k = entry_key64(a, Entry{E.key(tid), E.code(tid)});
  // the network moves the order keys alone: an entry's mass is a function of its estimate (the key's
  // high half), recomputed after the sort
  if (tid < np) {
    for (int size = 2; size <= np; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const bool up = (tid & size) == 0;
        unsigned long long ok;
        if (stride >= 32) {  // partner in another warp: through shared memory
          ks[tid] = k;
          asm volatile("bar.sync 1, %0;" ::"r"(np) : "memory");
          ok = ks[tid ^ stride];
          asm volatile("bar.sync 1, %0;" ::"r"(np) : "memory");
        } else {
          ok = __shfl_xor_sync(0xffffffffu, k, stride);
        }
        const bool lower = (tid & stride) == 0;
        if ((up == lower) ? (ok < k) : (ok > k)) k = ok;
      }
    }
  }
  const unsigned long long w = tid < n ? entry_mass(m, uint32_t(k >> 32)) : 0ull;  // sorted: valid first
  unsigned long long Z;
  const unsigned long long before = block_scan_u64(w, sm.red64, &Z);
  const unsigned long long T = ceil_p_times(Z, a.p_mant[step], a.p_shift[step]);
  // sorted position of the cut: the first with before + w >= T (none: keep everything)
  if (tid == 0) sm.bcast64[1] = ~0ull;
  __syncthreads();
  if (tid < n && before < T && before + w >= T) sm.bcast64[1] = k;
  __syncthreads();
  const unsigned long long cut = sm.bcast64[1];
  __syncthreads();
  return cut;
}

// The cut of one routing step: the largest 64-bit order key (e desc, start
// asc) that is kept.  kmin is the smallest key (largest estimate) of the step.
// Every thread returns the same value.
template <class View>
__device__ __noinline__ unsigned long long select_cut(const DecodeArgs& a, const View E, int64_t n, uint32_t kmin,
                                         DecSmem& sm, int h, int step) {
  const int tid = threadIdx.x, lane = tid & 31;
  if (a.p_all[step]) return ~0ull;
  const float m = desc_key_value(kmin);
  if (n <= kDecThreads) return select_cut_small(a, E, n, m, sm, step);

  // coarse histogram of the masses (and counts); total mass Z and the target T = ceil(p Z)
  for (int i = tid; i < kBins; i += kDecThreads) sm.hist[i] = 0ull;
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
    for (int u = 0; u < U; ++u) hist_add_warp(sm.hist, bin[u], w[u]);
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
  const unsigned long long T = ceil_p_times(Z, a.p_mant[step], a.p_shift[step]);  // keep while mass before < T
  unsigned long long below;
  const int cb = find_cut_bin(sm, 0ull, T, &below);
  if (cb < 0) return ~0ull;  // cannot happen for 0 < p < 1; keep everything
  // members of the coarse bin cb (the bin is monotone in the key: one contiguous key range)
  auto in_cb = [&](uint32_t k) { return coarse_bin(entry_gap(m, k)) == cb; };

  // fine histogram inside the cut coarse bin
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
        if (in_cb(k)) {
          bin[u] = fine_bin(entry_gap(m, k), cb);
          w[u] = entry_mass(m, k);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) hist_add_warp(sm.hist, bin[u], w[u]);
  }
  __syncthreads();
  unsigned long long below2;
  const int fb = find_cut_bin(sm, below, T, &below2);
  if (fb < 0) return ~0ull;
  auto in_cut = [&](uint32_t k) {  // a member of the cut fine bin
    const float x = entry_gap(m, k);
    return coarse_bin(x) == cb && fine_bin(x, cb) == fb;
  };

  // gather the entries around the cut
  if (tid == 0) sm.bcast32[1] = 0;
  __syncthreads();
  for (int i = tid; i < n32; i += kDecThreads) {
    const uint32_t k = E.key(i);
    if (in_cut(k)) {
      const int s = smem_inc(&sm.bcast32[1]);
      if (s < 32) {
        sm.cut_key[s] = entry_key64(a, Entry{k, E.code(i)});
        sm.cut_w[s] = entry_mass(m, k);
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
      smem_add_u64(&sm.hist[(k64 >> shift) & 255], entry_mass(m, k));
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

// ---------------------------------------------------------------- anchored histograms
// The scoring warps of step s >= 1 add every new entry's mass to a histogram
// of the head's step, anchored at r = the largest estimate of step s-1 (known
// before step s is scored): bin floor(32 x) of x = (r - e) + kAnchorSpan (the
// last bin open), mass exp(-(x - bin/32)) as a 2^-40 fixed-point integer
// (<= 2^40, exact order-independent sums).  A bin's mass relative to the
// anchor is its integer sum times anchored_scale(bin).  An estimate above
// r + kAnchorSpan sets the step's overflow flag; the select then recomputes
// the masses relative to the step's own max, as it does when r lies more
// than kAnchorFar above that max (the fixed point would lose the masses).
constexpr float kAnchorSpan = 8.f;
constexpr float kAnchorFar = 16.f;
__device__ __forceinline__ int anchored_bin(float r, uint32_t key, unsigned long long* w, float* t) {
  const float x = __fadd_rn(__fsub_rn(r, desc_key_value(key)), kAnchorSpan);
  if (!(x >= 0.f)) return -1;
  const int b = min(int(__fmul_rn(x, kBinScale)), kBins - 1);
  const float tt = __fsub_rn(x, __fmul_rn(float(b), 1.f / kBinScale));
  *t = tt;
  *w = __float2ull_rn(__fmul_rn(expf(-tt), 1099511627776.0f));  // 2^40
  return b;
}
__device__ __forceinline__ double anchored_scale(int b) {
  return exp(double(kAnchorSpan) - double(b) / double(kBinScale)) * 0x1p-40;
}
// sub-bin of t = x - bin/32 inside its bin: 1024 sub-bins of 1/32768, the last open
__device__ __forceinline__ int anchored_fine(float t) {
  return min(int(__fmul_rn(t, kBinScale * float(kBins))), kBins - 1);
}

// Block-wide exclusive scan of one double per thread, in a fixed order (so
// that every run gives the same sums); *total = the block total.
__device__ __forceinline__ double block_scan_f64(double v, double* red, double* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  double x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  double ex = __shfl_up_sync(0xffffffffu, x, 1);
  if (lane == 0) ex = 0.0;
  if (lane == 31) red[wid] = x;
  __syncthreads();
  // the warp totals, scanned across lanes in warp order
  double t = lane < kDecWarps ? red[lane] : 0.0;
#pragma unroll
  for (int off = 1; off < kDecWarps; off <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, t, off);
    if (lane >= off) t += y;
  }
  const double base = __shfl_sync(0xffffffffu, t, (wid + 31) & 31);
  *total = __shfl_sync(0xffffffffu, t, kDecWarps - 1);
  __syncthreads();
  return (wid > 0 ? base : 0.0) + ex;
}

// First of kBins per-thread-blocked bin masses (BPT consecutive bins per
// thread, exclusive prefix `before`) at which base + running mass reaches T:
// returns the bin and the mass before it (all threads); -1 if none does.
__device__ __forceinline__ int find_cut_bin_f64(DecSmem& sm, const double* m, double before, double T,
                                                double* below_out) {
  constexpr int BPT = kBins / kDecThreads;
  const int tid = threadIdx.x;
  if (tid == 0) sm.bcast32[0] = -1;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < BPT; ++k) {
    if (before < T && before + m[k] >= T) {
      sm.bcast32[0] = tid * BPT + k;
      sm.bcast64[0] = (unsigned long long)__double_as_longlong(before);
    }
    before += m[k];
  }
  __syncthreads();
  const int bin = sm.bcast32[0];
  *below_out = __longlong_as_double((long long)sm.bcast64[0]);
  __syncthreads();
  return bin;
}

// Bin of a key for anchor r (the anchored_bin bin alone, no mass), and the
// bin's sub-bin, as monotone non-decreasing functions of the key: -1 for an
// estimate above the anchor span.
__device__ __forceinline__ int anchored_bin_of(float r, uint32_t key) {
  const float x = __fadd_rn(__fsub_rn(r, desc_key_value(key)), kAnchorSpan);
  if (!(x >= 0.f)) return -1;
  return min(int(__fmul_rn(x, kBinScale)), kBins - 1);
}
// (coarse bin, sub-bin) ordered as one number: coarse * kBins + fine
__device__ __forceinline__ long long anchored_code_of(float r, uint32_t key) {
  const float x = __fadd_rn(__fsub_rn(r, desc_key_value(key)), kAnchorSpan);
  if (!(x >= 0.f)) return -1;
  const int b = min(int(__fmul_rn(x, kBinScale)), kBins - 1);
  const float t = __fsub_rn(x, __fmul_rn(float(b), 1.f / kBinScale));
  return (long long)b * kBins + anchored_fine(t);
}


// The cut of a step from its anchored histogram (kBins sums; ghist is the
// caller's shared-memory copy in sm.hist, read before sm.hist is reused): the
// coarse cut bin from the histogram alone; one pass over the keys for the
// sub-bin histogram of that bin's members, one more to gather the members of
// the cut sub-bin, which are ordered by (e desc, start asc).  Membership is
// tested on each key's (bin, sub-bin), both monotone in the key, so the
// members are exactly the keys of one contiguous key range.  Passes read four
// keys per lane and do the mass work only for members.  Every thread returns
// the same value.
template <class View>
__device__ __noinline__ unsigned long long select_cut_anchored(const DecodeArgs& a, const View E, int64_t n,
                                                               float r, const unsigned long long* ghist,
                                                               DecSmem& sm, int h, int step) {
  const int tid = threadIdx.x;
  constexpr int BPT = kBins / kDecThreads;
  double* red = reinterpret_cast<double*>(sm.red64);
  const double p = ldexp(double(a.p_mant[step]), -a.p_shift[step]);
  double mb[BPT], loc = 0.0;
#pragma unroll
  for (int k = 0; k < BPT; ++k) {
    const int bin = tid * BPT + k;
    mb[k] = double(ghist[bin]) * anchored_scale(bin);
    loc += mb[k];
  }
  double Z;
  const double before = block_scan_f64(loc, red, &Z);
  const double T = p * Z;
  double below_c;
  const int cb = find_cut_bin_f64(sm, mb, before, T, &below_c);
  if (cb < 0) return ~0ull;  // rounding kept T out of reach: keep everything
  const double sc = anchored_scale(cb);
  for (int i = tid; i < kBins; i += kDecThreads) sm.hist[i] = 0ull;
  __syncthreads();
  const int n32 = int(n);
  // sub-bin histogram of the members (exact integer masses), four keys per lane
  auto keys4 = [&](int i0, uint32_t* k) {  // keys i0 .. i0+3 (past n: 0xffffffff, never a member)
    if (i0 + 4 <= E.nc) {
      const uint4 v = *reinterpret_cast<const uint4*>(E.ck + i0);
      k[0] = v.x;
      k[1] = v.y;
      k[2] = v.z;
      k[3] = v.w;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) k[u] = i0 + u < n32 ? E.key(i0 + u) : 0xffffffffu;
    }
  };
  for (int b0 = 0; b0 < n32; b0 += 4 * kDecThreads) {  // every lane of a warp takes part in each round
    const int i0 = b0 + 4 * tid;
    uint32_t k[4];
    keys4(i0, k);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int fb = -1;
      unsigned long long w = 0;
      if (anchored_bin_of(r, k[u]) == cb) {  // a member of the coarse bin
        float t;
        anchored_bin(r, k[u], &w, &t);
        fb = anchored_fine(t);
      }
      hist_add_warp(sm.hist, fb, w);
    }
  }
  __syncthreads();
  double fm[BPT];
  loc = 0.0;
#pragma unroll
  for (int k = 0; k < BPT; ++k) {
    fm[k] = double(sm.hist[tid * BPT + k]) * sc;
    loc += fm[k];
  }
  double FZ;
  const double fbefore = block_scan_f64(loc, red, &FZ);
  double below_f;
  int fbin = find_cut_bin_f64(sm, fm, below_c + fbefore, T, &below_f);
  if (fbin < 0) {  // rounding: the sub-bins fell short of T; take the last non-empty one
    if (tid == 0) sm.bcast32[2] = -1;
    __syncthreads();
    for (int k = 0; k < BPT; ++k)
      if (sm.hist[tid * BPT + k] != 0ull) smem_max_s32(&sm.bcast32[2], tid * BPT + k);
    __syncthreads();
    fbin = sm.bcast32[2];
    if (fbin < 0) return ~0ull;
    unsigned long long pre = 0;
    for (int k = 0; k < fbin; ++k) pre += sm.hist[k];
    below_f = below_c + double(pre) * sc;
    __syncthreads();
  }
  const long long fcode = (long long)cb * kBins + fbin;  // (coarse bin, sub-bin) of the cut
  if (tid == 0) sm.bcast32[1] = 0;
  __syncthreads();
  // gather the members of the cut sub-bin
  for (int i0 = 4 * tid; i0 < n32; i0 += 4 * kDecThreads) {
    uint32_t k[4];
    keys4(i0, k);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (anchored_code_of(r, k[u]) == fcode) {
        unsigned long long w;
        float t;
        anchored_bin(r, k[u], &w, &t);
        const int sl = smem_inc(&sm.bcast32[1]);
        if (sl < 32) {
          sm.cut_key[sl] = entry_key64(a, Entry{k[u], E.code(i0 + u)});
          sm.cut_w[sl] = w;
        }
      }
    }
  }
  __syncthreads();
  const int cnt = sm.bcast32[1];
  if (cnt <= 32) {
    if (tid < 32) {
      unsigned long long k = tid < cnt ? sm.cut_key[tid] : ~0ull;
      unsigned long long w = tid < cnt ? sm.cut_w[tid] : 0ull;
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          const unsigned long long ok = __shfl_xor_sync(0xffffffffu, k, stride);
          const unsigned long long ow = __shfl_xor_sync(0xffffffffu, w, stride);
          const bool up = ((tid & size) == 0);
          const bool lower = ((tid & stride) == 0);
          const bool swap = (up == lower) ? (ok < k) : (ok > k);
          if (swap) {
            k = ok;
            w = ow;
          }
        }
      }
      unsigned long long c = w;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, c, off);
        if (tid >= off) c += y;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, tid < cnt && below_f + double(c) * sc >= T);
      const int first = hit ? __ffs(hit) - 1 : max(cnt - 1, 0);
      const unsigned long long cut = __shfl_sync(0xffffffffu, k, first);
      if (tid == 0) sm.bcast64[1] = cnt > 0 ? cut : ~0ull;
    }
    __syncthreads();
    return sm.bcast64[1];
  }
  // Many members share the cut sub-bin (exact ties or near-ties): radix
  // select on the 64-bit order key, 8 bits per pass, over those members.
  unsigned long long prefix = 0, acc = 0;  // acc: exact mass of the members before the prefix's range
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = tid; i < 256; i += kDecThreads) sm.hist[i] = 0ull;
    __syncthreads();
    for (int i = tid; i < n32; i += kDecThreads) {
      const uint32_t k = E.key(i);
      if (anchored_code_of(r, k) != fcode) continue;
      unsigned long long w;
      float t;
      anchored_bin(r, k, &w, &t);
      const unsigned long long k64 = entry_key64(a, Entry{k, E.code(i)});
      if (pass > 0 && (k64 >> (shift + 8)) != (prefix >> (shift + 8))) continue;
      smem_add_u64(&sm.hist[(k64 >> shift) & 255], w);
    }
    __syncthreads();
    if (tid < 32) {
      unsigned long long loc8 = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) loc8 += sm.hist[tid * 8 + k];
      unsigned long long c = loc8;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, c, off);
        if (tid >= off) c += y;
      }
      unsigned long long bef = acc + c - loc8;
      int digit = -1, last = -1;
      unsigned long long dbef = 0, lbef = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const unsigned long long hb = sm.hist[tid * 8 + k];
        if (digit < 0 && below_f + double(bef + hb) * sc >= T) {
          digit = tid * 8 + k;
          dbef = bef;
        }
        if (hb) {
          last = tid * 8 + k;
          lbef = bef;
        }
        bef += hb;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, digit >= 0);
      const unsigned any = __ballot_sync(0xffffffffu, last >= 0);
      int dg;
      unsigned long long db;
      if (hit) {
        const int src = __ffs(hit) - 1;
        dg = __shfl_sync(0xffffffffu, digit, src);
        db = __shfl_sync(0xffffffffu, dbef, src);
      } else {  // rounding: fall back to the last non-empty digit
        const int src = any ? 31 - __clz(any) : 31;
        dg = __shfl_sync(0xffffffffu, last, src);
        db = __shfl_sync(0xffffffffu, lbef, src);
        if (!any) {
          dg = 255;
          db = acc;
        }
      }
      if (tid == 0) {
        sm.bcast64[2] = prefix | (uint64_t(dg) << shift);
        sm.bcast64[3] = db;
      }
    }
    __syncthreads();
    prefix = sm.bcast64[2];
    acc = sm.bcast64[3];
    __syncthreads();
  }
  return prefix;
}

// Inclusive prefix of per-head counts held in pref[1..nh] (pref[0] = 0), NT
// threads; returns the total.
template <int NT>
__device__ __forceinline__ long long build_prefix(long long* pref, unsigned long long* red64, int nh) {
  if (nh <= 32) {  // one warp scans with shuffles; one CTA barrier (red64[0] carries the total)
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      long long v = lane < nh ? pref[1 + lane] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += y;
      }
      if (lane < nh) pref[1 + lane] = v;
      if (lane == 0) pref[0] = 0;
      if (lane == 31) red64[0] = (unsigned long long)v;
    }
    __syncthreads();
    return (long long)red64[0];
  }
  long long carry = 0;
  for (int base = 0; base < nh; base += NT) {
    const int i = base + threadIdx.x;
    const unsigned long long v = i < nh ? (unsigned long long)pref[1 + i] : 0ull;
    unsigned long long tot;
    const unsigned long long ex = block_scan_u64<NT / 32>(v, red64, &tot);
    if (i < nh) pref[1 + i] = carry + (long long)(ex + v);
    carry += (long long)tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) pref[0] = 0;
  __syncthreads();
  return carry;
}

// Head owning work item i: the largest h with pref[h] <= i.
__device__ __forceinline__ int owner_of(const long long* pref, int nh, long long i) {
  int lo = 0, hi = nh - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pref[mid] <= i) lo = mid; else hi = mid - 1;
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

// ---------------------------------------------------------------- bulk copies
// A node record is fetched with one bulk copy (cp.async.bulk, no multicast)
// issued by one lane; completion is counted in bytes on a per-slot mbarrier.
__device__ __forceinline__ unsigned smem_u32(const void* p) { return unsigned(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void mbar_init(unsigned long long* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void bulk_load(void* dst, const void* src, unsigned bytes, unsigned long long* bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Orders this thread's earlier shared-memory reads before later bulk-copy writes.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------- tensor-core estimate (bf16)
// The q operand of the estimate, as B fragments of m16n8k16 (column 0 = q, the
// other columns zero).  The k order of each k-step is a permutation of the
// dimensions chosen so that a lane's A words are whole 16-byte chunks of a
// record row: lane (g = lane/4, t = lane%4) takes chunk q_chunk(t, c) of its
// rows as its c-th chunk (c < CPL = D/32), which feeds k-steps 2c and 2c+1,
// dims 0-3 the first and 4-7 the second, as (k 2t, 2t+1) and (k 2t+8, 2t+9).
// The same permutation applied to q leaves the dot product unchanged.  Two
// chunk orders: interleaved (chunk c*4 + t: the four lanes of a row read 64
// contiguous bytes, so the two rows of a quarter-warp meet in at most two-way
// shared-memory bank conflicts), used for the bf16 slope rows; blocked (chunk
// t*CPL + c: a lane's chunks contiguous), used for the FP4 router rows, whose
// packed codes a lane reads as one 16-byte word.
template <int D, bool kInterleave>
__device__ __forceinline__ int q_chunk(int t, int c) {
  return kInterleave ? c * 4 + t : t * (D / 32) + c;
}
template <int D, bool kInterleave = true>
__device__ __forceinline__ void q_fragments(const __nv_bfloat16* q, uint32_t (&qf)[D / 16][2], int lane) {
  constexpr int CPL = D / 32;
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (g == 0) v = *reinterpret_cast<const uint4*>(q + q_chunk<D, kInterleave>(t, c) * 8);
    qf[2 * c][0] = v.x;
    qf[2 * c][1] = v.y;
    qf[2 * c + 1][0] = v.z;
    qf[2 * c + 1][1] = v.w;
  }
}

// e = max_j (b_j + q.mu_j / sqrt d) of a bf16 record in shared memory: the
// R x D slope rows times q on the tensor cores (fp32 accumulation), 16 rows
// per m-tile; every lane returns the estimate.
template <int D>
__device__ __forceinline__ float score_record_mma(const unsigned char* rec, int R, float inv_sqrt_d,
                                                  const uint32_t (&qf)[D / 16][2], int lane) {
  constexpr int CPL = D / 32;
  const int g = lane >> 2, t = lane & 3;
  const float* bias = reinterpret_cast<const float*>(rec + size_t(R) * D * 2);
  float best = -INFINITY;
  for (int m0 = 0; m0 < R; m0 += 16) {
    const int r0 = min(m0 + g, R - 1), r1 = min(m0 + g + 8, R - 1);  // rows past R: any valid row, masked below
    const unsigned char* p0 = rec + size_t(r0) * D * 2 + t * 16;
    const unsigned char* p1 = rec + size_t(r1) * D * 2 + t * 16;
    // four independent accumulators: chunk c's two k-steps go to
    // cc[2 (c & 1)] and cc[2 (c & 1) + 1], chains of CPL / 2 products each
    float cc[4][4] = {};
#pragma unroll
    for (int c = 0; c < CPL; ++c) {  // chunk q_chunk<D, true>(t, c) = c*4 + t
      const uint4 x0 = *reinterpret_cast<const uint4*>(p0 + c * 64);
      const uint4 x1 = *reinterpret_cast<const uint4*>(p1 + c * 64);
      const uint32_t a0[4] = {x0.x, x1.x, x0.y, x1.y};
      const uint32_t a1[4] = {x0.z, x1.z, x0.w, x1.w};
      mma_bf16_16816(cc[2 * (c & 1)], a0, qf[2 * c]);
      mma_bf16_16816(cc[2 * (c & 1) + 1], a1, qf[2 * c + 1]);
    }
    if (t == 0) {
      const int j0 = m0 + g, j1 = m0 + g + 8;
      const float s0 = (cc[0][0] + cc[1][0]) + (cc[2][0] + cc[3][0]);
      const float s1 = (cc[0][2] + cc[1][2]) + (cc[2][2] + cc[3][2]);
      if (j0 < R) best = fmaxf(best, fmaf(s0, inv_sqrt_d, bias[j0]));
      if (j1 < R) best = fmaxf(best, fmaf(s1, inv_sqrt_d, bias[j1]));
    }
  }
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, off));
  return best;
}

// The q operand for FP4 router records: the bf16 fragments of q_fragments in
// the blocked chunk order, converted to f16 (exact for the normal f16 range).
template <int D>
__device__ __forceinline__ void q_fragments_f16(const __nv_bfloat16* q, uint32_t (&qf)[D / 16][2], int lane) {
  q_fragments<D, false>(q, qf, lane);
#pragma unroll
  for (int k = 0; k < D / 16; ++k)
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float lo = __uint_as_float(qf[k][u] << 16), hi = __uint_as_float(qf[k][u] & 0xffff0000u);
      const __half2 h = __floats2half2_rn(lo, hi);
      qf[k][u] = *reinterpret_cast<const uint32_t*>(&h);
    }
}

// e = max_j (b_j + q.mu_j / sqrt d) of an FP4 router record in shared memory:
// the lane's 4-bit codes of its two rows are turned into f16 (exact) and
// multiplied by their groups' e4m3 scales (exact in f16), then fed to the
// tensor cores in the same operand layout as score_record_mma (f16, fp32
// accumulation); every lane returns the estimate.
template <int D>
__device__ __forceinline__ float score_record_fp4(const unsigned char* rec, int R, float inv_sqrt_d,
                                                  const uint32_t (&qf)[D / 16][2], int lane) {
  constexpr int CPL = D / 32;  // 8-dimension chunks per lane
  const int g = lane >> 2, t = lane & 3;
  const unsigned char* scales = rec + size_t(R) * (D / 2);
  const float* bias = reinterpret_cast<const float*>(rec + size_t(R) * (D / 2 + D / 16));
  float best = -INFINITY;
  for (int m0 = 0; m0 < R; m0 += 16) {
    const int r0 = min(m0 + g, R - 1), r1 = min(m0 + g + 8, R - 1);  // rows past R: masked below
    uint32_t w0[CPL], w1[CPL];  // 4 code bytes (8 dimensions) per chunk
    uint32_t s0, s1;            // the rows' scales of the lane's groups, as f16x2
    if constexpr (D == 128) {
      const uint4 v0 = *reinterpret_cast<const uint4*>(rec + size_t(r0) * (D / 2) + t * 16);
      const uint4 v1 = *reinterpret_cast<const uint4*>(rec + size_t(r1) * (D / 2) + t * 16);
      w0[0] = v0.x; w0[1] = v0.y; w0[2] = v0.z; w0[3] = v0.w;
      w1[0] = v1.x; w1[1] = v1.y; w1[2] = v1.z; w1[3] = v1.w;
      s0 = e4m3x2_to_f16x2(*reinterpret_cast<const unsigned short*>(scales + size_t(r0) * (D / 16) + 2 * t));
      s1 = e4m3x2_to_f16x2(*reinterpret_cast<const unsigned short*>(scales + size_t(r1) * (D / 16) + 2 * t));
    } else {
      const uint2 v0 = *reinterpret_cast<const uint2*>(rec + size_t(r0) * (D / 2) + t * 8);
      const uint2 v1 = *reinterpret_cast<const uint2*>(rec + size_t(r1) * (D / 2) + t * 8);
      w0[0] = v0.x; w0[1] = v0.y;
      w1[0] = v1.x; w1[1] = v1.y;
      const uint32_t b0 = scales[size_t(r0) * (D / 16) + t], b1 = scales[size_t(r1) * (D / 16) + t];
      s0 = e4m3x2_to_f16x2(b0 | (b0 << 8));
      s1 = e4m3x2_to_f16x2(b1 | (b1 << 8));
    }
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      // chunk c lies in group c/2 of the lane's (D = 128) or in its only group (D = 64)
      const uint32_t sel = (D == 128 && c >= 2) ? 0x3232u : 0x1010u;
      const uint32_t S0 = __byte_perm(s0, s0, sel), S1 = __byte_perm(s1, s1, sel);
      uint32_t x0[4], x1[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        x0[q] = hmul2_u32(e2m1x2_to_f16x2(w0[c] >> (8 * q)), S0);
        x1[q] = hmul2_u32(e2m1x2_to_f16x2(w1[c] >> (8 * q)), S1);
      }
      const uint32_t a0[4] = {x0[0], x1[0], x0[1], x1[1]};
      const uint32_t a1[4] = {x0[2], x1[2], x0[3], x1[3]};
      mma_f16_16816(c0, a0, qf[2 * c]);
      mma_f16_16816(c1, a1, qf[2 * c + 1]);
    }
    if (t == 0) {
      const int j0 = m0 + g, j1 = m0 + g + 8;
      if (j0 < R) best = fmaxf(best, fmaf(c0[0] + c1[0], inv_sqrt_d, bias[j0]));
      if (j1 < R) best = fmaxf(best, fmaf(c0[2] + c1[2], inv_sqrt_d, bias[j1]));
    }
  }
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, off));
  return best;
}

// Estimate of a node whose record sits in shared memory (whole warp; the
// lane's q slice covers elements [cl*EPC, cl*EPC+EPC), cl = lane % CPR).  Up
// to kG reference rows per lane are in flight at once: their partial dot
// products are formed independently, then reduced over the CPR lanes of each
// row together, so that the shuffles of different rows overlap.  The
// arithmetic (FMA order inside a lane, the butterfly over lanes) is the same
// for every row count.
template <typename T, int D>
__device__ __forceinline__ float score_record_smem(const unsigned char* rec, int R, float inv_sqrt_d,
                                                   const float* qs, int lane) {
  constexpr int EPC = 16 / sizeof(T);
  constexpr int CPR = D * sizeof(T) / 16;
  constexpr int RPI = 32 / CPR;
  constexpr int kG = 8;
  const float* bias = reinterpret_cast<const float*>(rec + size_t(R) * D * sizeof(T));
  const int sub = lane / CPR, cl = lane % CPR;
  float best = -INFINITY;
  for (int j0 = 0; j0 < R; j0 += RPI * kG) {
    float part[kG];
#pragma unroll
    for (int g = 0; g < kG; ++g) {
      const int j = j0 + g * RPI + sub;
      part[g] = 0.f;
      if (j < R) {
        const uint4 v = *reinterpret_cast<const uint4*>(rec + (size_t(j) * CPR + cl) * 16);
        float x[EPC];
        unpack16<T>(v, x);
#pragma unroll
        for (int i = 0; i < EPC; ++i) part[g] = fmaf(x[i], qs[i], part[g]);
      }
    }
#pragma unroll
    for (int off = CPR / 2; off > 0; off >>= 1) {
#pragma unroll
      for (int g = 0; g < kG; ++g) part[g] += __shfl_xor_sync(0xffffffffu, part[g], off);
    }
#pragma unroll
    for (int g = 0; g < kG; ++g) {
      const int j = j0 + g * RPI + sub;
      if (j < R) best = fmaxf(best, fmaf(part[g], inv_sqrt_d, bias[j]));
    }
  }
#pragma unroll
  for (int off = 16; off >= CPR; off >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, off));
  return best;
}

// ---------------------------------------------------------------- launch overlap
// Every decode kernel is launched with programmatic stream serialization: it
// may start while the kernel before it finishes, lets the next one start too,
// and waits for the one before to complete (memory visible) before it reads
// anything that kernel wrote.
__device__ __forceinline__ void pdl_wait_and_release() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// The kernel arguments copied into shared memory by the whole CTA (ends with
// a CTA barrier).  The select code runs in non-inlined functions that reach
// the arguments through a reference: with the copy, that reference points to
// shared memory rather than into the parameter space, and the per-call
// context each function builds from it stays in registers (no stack frame).
__device__ __forceinline__ void stage_args(const DecodeArgs& src, DecodeArgs* dst) {
  static_assert(sizeof(DecodeArgs) % 4 == 0, "argument block of whole words");
  const uint32_t* from = reinterpret_cast<const uint32_t*>(&src);
  uint32_t* to = reinterpret_cast<uint32_t*>(dst);
  for (int i = threadIdx.x; i < int(sizeof(DecodeArgs) / 4); i += blockDim.x) to[i] = from[i];
  __syncthreads();
}

// ---------------------------------------------------------------- per-call context
// The scratch regions of one decode call and the views of them every phase uses.
template <typename T, int D>
struct Ctx {
  const DecodeArgs& a;
  int nh;  // heads of this call
  int mh;  // heads the scratch is laid out for (every call uses the same offsets)
  int64_t cap4, bm_words;
  __device__ explicit Ctx(const DecodeArgs& args)
      : a(args), nh(args.nheads), mh(args.max_heads), cap4((args.cap_sel + 3) & ~int64_t(3)),
        bm_words(decode_bitmap_words(args.cap_sel)) {}
  // per-head workspace: step keys [2][cap4], step codes [2][cap4] (parity buffers: step s in s & 1),
  // anchored histograms [2][kBins], units of the next scoring phase [cap4], kept leaves [cap_list]
  __device__ char* ws(int h) const { return a.ws + uint64_t(h) * a.ws_per_bh; }
  __device__ uint32_t* keysP(int h, int par) const { return reinterpret_cast<uint32_t*>(ws(h) + par * cap4 * 4); }
  __device__ uint32_t* codesP(int h, int par) const {
    return reinterpret_cast<uint32_t*>(ws(h) + (2 + par) * cap4 * 4);
  }
  __device__ unsigned long long* histP(int h, int par) const {
    return reinterpret_cast<unsigned long long*>(ws(h) + 4 * cap4 * 4 + par * kBins * 8);
  }
  __device__ uint32_t* units(int h) const { return reinterpret_cast<uint32_t*>(ws(h) + 4 * cap4 * 4 + 2 * kBins * 8); }
  __device__ uint32_t* leaves(int h) const {
    return reinterpret_cast<uint32_t*>(ws(h) + 5 * cap4 * 4 + 2 * kBins * 8);
  }
  // head states, then one leaf bitmap per head (one region, zero between calls)
  __device__ HeadState* hstate(int h) const { return reinterpret_cast<HeadState*>(a.flow) + h; }
  __device__ uint32_t* bitmap(int h) const {
    return reinterpret_cast<uint32_t*>(a.flow + size_t(mh) * sizeof(HeadState)) + h * bm_words;
  }
  // the lane's q slice for the FMA estimates: elements [cl*EPC, cl*EPC+EPC), cl = lane % CPR
  __device__ void q_slice(int h, float* qs) const {
    constexpr int EPC = 16 / sizeof(T);
    constexpr int CPR = D * sizeof(T) / 16;
    const T* q = static_cast<const T*>(a.Q) + size_t(h) * D + ((threadIdx.x & 31) % CPR) * EPC;
    unpack16<T>(*reinterpret_cast<const uint4*>(q), qs);
  }
};

// ---------------------------------------------------------------- select
// One head, whole CTA: the cut of step s (small path, anchored histogram or
// the in-CTA histograms), then the kept entries in entry order, split by
// level: kept non-leaves become the units of step s+1 (unit u's b children
// are scored into positions u*b .. u*b+b-1 of step s+1), kept level-1 blocks
// are appended to the head's leaf list.  The head's state and the step's
// first kSpecEnt keys and codes are fetched together; a larger step's other
// keys and codes follow once its size is known.
template <typename T, int D>
__device__ __noinline__ void export_kept(const DecodeArgs& a, uint32_t* red32, int h);

template <typename T, int D>
__device__ __noinline__ void select_head(const DecodeArgs& a, DecSmem& sm, int h, int s) {
  const Ctx<T, D> c(a);
  const int tid = threadIdx.x;
  const int par = s & 1;
  const bool last = s + 1 == a.n_steps;
  const int b = a.t.block;
  HeadState* hs = c.hstate(h);
  const uint32_t* gk = c.keysP(h, par);
  const uint32_t* gc = c.codesP(h, par);
  uint32_t* ck = reinterpret_cast<uint32_t*>(sm.u);
  uint32_t* cc = ck + kCacheEnt;
  const int spec = int(min64(kSpecEnt, c.cap4));
  for (int v = tid; v < spec / 4; v += kDecThreads) {
    cp_async16(ck + 4 * v, gk + 4 * v);
    cp_async16(cc + 4 * v, gc + 4 * v);
  }
  if (s >= 1) {  // the step's anchored histogram, for the anchored cut (every other cut rewrites sm.hist)
    const unsigned long long* gh = c.histP(h, par);
    for (int v = tid; v < kBins / 2; v += kDecThreads) cp_async16(sm.hist + 2 * v, gh + 2 * v);
  }
  cp_async_commit();
  // the next step's histogram cleared while the copies are in flight (step s-1 wrote and read it; step
  // s+1's scoring writes it after this kernel)
  if (!last) {
    unsigned long long* nhist = c.histP(h, par ^ 1);
    for (int i = tid; i < kBins; i += kDecThreads) nhist[i] = 0ull;
  }
  // step 0 starts the head's counters afresh
  const long long n = s == 0 ? (long long)a.n_roots : min64(max64(__ldcg(&hs->n[par]), 0), a.cap_sel);
  const uint32_t kmin = ~__ldcg(&hs->kinv[par]);  // smallest key (largest estimate) of the step
  const float anchor_h = __ldcg(&hs->anchor);
  const int ovf = __ldcg(&hs->ovf[par]);
  const long long scored0 = s == 0 ? 0 : __ldcg(&hs->scored);
  const long long leaves0 = s == 0 ? 0 : min64(max64(__ldcg(&hs->n_leaf), 0), a.cap_list);
  const int leaf0_in = s == 0 ? 0 : __ldcg(&hs->leaf0);
  const int steps0 = s == 0 ? 0 : __ldcg(&hs->steps);
  const int ncache = int(min64(n, kCacheEnt));
  for (int v = spec / 4 + tid; v < (ncache + 3) / 4; v += kDecThreads) {
    cp_async16(ck + 4 * v, gk + 4 * v);
    cp_async16(cc + 4 * v, gc + 4 * v);
  }
  cp_async_commit();
  cp_async_wait(0);
  __syncthreads();
  const StepView E{ck, cc, ncache, gk, gc};
  if (a.scored) {  // codes of the scored nodes
    int32_t* out = a.scored + size_t(h) * a.scored_cap;
    for (long long i = tid; i < n; i += kDecThreads)
      if (scored0 + i < a.scored_cap) out[scored0 + i] = int32_t(E.code(i));
  }
  const float m = desc_key_value(kmin);
  unsigned long long cut = ~0ull;
  if (!a.p_all[s] && n > 0) {
    if (n <= kDecThreads) cut = select_cut_small(a, E, n, m, sm, s);
    else if (s >= 1 && !ovf && __fsub_rn(anchor_h, m) <= kAnchorFar)
      cut = select_cut_anchored(a, E, n, anchor_h, sm.hist, sm, h, s);
    else cut = select_cut(a, E, n, kmin, sm, h, s);
  }
  // the kept entries (order key <= cut) in entry order.  A round covers two
  // sub-rounds of 4 * kDecThreads entries, four per thread each (16-byte
  // loads); one block scan per round of four 16-bit counts packed in 64 bits
  // (units and leaves of each sub-round) gives every position, so the lists
  // stay in entry order.  Kept non-leaves go to the units list (the next
  // scoring step checks each code before it reads a record); a kept level-1
  // block is listed only if its index lies in the level (it addresses the
  // bitmap and the attention's key ranges).
  const uint32_t cut32 = uint32_t(cut >> 32);
  const int n32 = int(n);
  const uint64_t nl1 = uint64_t(a.nl[1]);
  uint32_t* un = c.units(h);
  uint32_t* lv = c.leaves(h);
  uint32_t* bm = c.bitmap(h);
  long long nu = 0, nlf = 0;
  int leaf0 = 0;
  constexpr int kSub = 4 * kDecThreads;  // entries of a sub-round
  for (int base = 0; base < n32; base += 2 * kSub) {
    uint32_t k[2][4], cd[2][4];
    unsigned kb[2] = {0u, 0u}, lb[2] = {0u, 0u};
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (r == 1 && base + kSub >= n32) break;  // (uniform) no entry in the second sub-round
      const int i0 = base + r * kSub + 4 * tid;
      if (i0 + 4 <= ncache) {
        const uint4 kv = *reinterpret_cast<const uint4*>(ck + i0);
        const uint4 cv = *reinterpret_cast<const uint4*>(cc + i0);
        k[r][0] = kv.x; k[r][1] = kv.y; k[r][2] = kv.z; k[r][3] = kv.w;
        cd[r][0] = cv.x; cd[r][1] = cv.y; cd[r][2] = cv.z; cd[r][3] = cv.w;
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          k[r][u] = i0 + u < n32 ? E.key(i0 + u) : 0xffffffffu;
          cd[r][u] = i0 + u < n32 ? E.code(i0 + u) : 0u;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool kp = i0 + u < n32 &&
                        (k[r][u] < cut32 || (k[r][u] == cut32 && entry_key64(a, Entry{k[r][u], cd[r][u]}) <= cut));
        const bool leaf = code_level(cd[r][u]) == 1;
        if (kp && (!leaf || uint64_t(code_index(cd[r][u])) < nl1)) {
          kb[r] |= 1u << u;
          if (leaf) lb[r] |= 1u << u;
        }
      }
    }
    // packed counts: leaves / units of sub-round 0 in bits 0-15 / 16-31, of sub-round 1 in 32-47 / 48-63
    const unsigned long long mine = (unsigned long long)__popc(lb[0]) | (unsigned long long)__popc(kb[0] & ~lb[0]) << 16 |
                                    (unsigned long long)__popc(lb[1]) << 32 |
                                    (unsigned long long)__popc(kb[1] & ~lb[1]) << 48;
    unsigned long long tot;
    const unsigned long long ex = block_scan_u64(mine, sm.red64, &tot);
    auto field = [](unsigned long long v, int f) { return (long long)((v >> (16 * f)) & 0xffffull); };
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (!kb[r]) continue;
      // sub-round 1 starts after every kept entry of sub-round 0
      long long pu = nu + field(ex, 2 * r + 1) + (r ? field(tot, 1) : 0);
      long long pl = leaves0 + nlf + field(ex, 2 * r) + (r ? field(tot, 0) : 0);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (!((kb[r] >> u) & 1u)) continue;
        if ((lb[r] >> u) & 1u) {
          const uint32_t li = code_index(cd[r][u]);
          if (pl < a.cap_list) lv[pl] = li;
          ++pl;
          leaf0 |= li == 0u ? 1 : 0;
          if (a.kept) atomicOr(bm + (li >> 5), 1u << (li & 31u));
        } else {
          un[pu++] = cd[r][u];
        }
      }
    }
    nu += field(tot, 1) + field(tot, 3);
    nlf += field(tot, 0) + field(tot, 2);
  }
  const int any_leaf0 = __syncthreads_or(leaf0);
  // state for the next step: its anchor = this step's max
  if (tid == 0) {
    long long U = nu, NL = leaves0 + nlf;
    if (U * b > a.cap_sel) {
      raise_status(a.t.status, ZHA_ERR_CAPACITY);
      U = a.cap_sel / b;
    }
    if (NL > a.cap_list) {
      raise_status(a.t.status, ZHA_ERR_CAPACITY);
      NL = a.cap_list;
    }
    hs->units = U;
    hs->n[par ^ 1] = U * b;
    hs->n_leaf = NL;
    hs->leaf0 = leaf0_in | any_leaf0;
    hs->anchor = m;
    hs->kinv[par ^ 1] = 0u;
    hs->ovf[par ^ 1] = 0;
    hs->scored = scored0 + n;
    hs->steps = steps0 + (n > 0 ? 1 : 0);
    if (last) {  // the next decode's first step finds its extremes cleared
      hs->kinv[par] = 0u;
      hs->ovf[par] = 0;
    }
  }
  if (last && a.kept) {
    __threadfence();
    __syncthreads();
    export_kept<T, D>(a, sm.red32, h);
  }
}

// ---------------------------------------------------------------- kept export
// The head's kept leaves in ascending block order from its bitmap (every
// select of a call with the export sets the bits of the leaves it keeps),
// which it leaves zeroed.  Each warp owns a contiguous run of words: counts,
// one scan over warps, then writes.
template <typename T, int D>
__device__ __noinline__ void export_kept(const DecodeArgs& a, uint32_t* red32, int h) {
  const Ctx<T, D> c(a);
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  uint32_t* bm = c.bitmap(h);
  const long long nw = min64((a.nl[1] + 31) / 32, c.bm_words);
  const long long wseg = (nw + kDecWarps - 1) / kDecWarps;
  const long long w_lo = min64(nw, wid * wseg), w_hi = min64(nw, w_lo + wseg);
  uint32_t cnt = 0;
  for (long long wi = w_lo + lane; wi < w_hi; wi += 32) cnt += __popc(__ldcg(bm + wi));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
  if (lane == 0) red32[wid] = cnt;
  __syncthreads();
  long long pos = 0;
  for (int w = 0; w < wid; ++w) pos += red32[w];
  __syncthreads();
  int32_t* out = a.kept + size_t(h) * a.kept_stride;
  for (long long wb = w_lo; wb < w_hi; wb += 32) {
    const long long wi = wb + lane;
    uint32_t bits = wi < w_hi ? __ldcg(bm + wi) : 0u;
    const uint32_t pc = __popc(bits);
    uint32_t ex = pc;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, ex, off);
      if (lane >= off) ex += y;
    }
    const uint32_t wtot = __shfl_sync(0xffffffffu, ex, 31);
    long long p = pos + ex - pc;
    if (bits) bm[wi] = 0u;
    while (bits) {
      const uint32_t idx = uint32_t(wi) * 32u + uint32_t(__ffs(bits) - 1);
      bits &= bits - 1u;
      if (p < a.kept_stride) out[p] = int32_t(idx);
      ++p;
    }
    pos += wtot;
  }
}

// One CTA per head.
template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads, 1) select_kernel(const __grid_constant__ DecodeArgs a_param, int s) {
  pdl_wait_and_release();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>(smem_raw);
  stage_args(a_param, &sm.args);
  const DecodeArgs& a = sm.args;
  for (int h = blockIdx.x; h < a.nheads; h += gridDim.x) {
    select_head<T, D>(a, sm, h, s);
    __syncthreads();
  }
}

// ---------------------------------------------------------------- scoring phase
// Step s's entries: the roots (s = 0, root i at position i) or the children of
// step s-1's kept non-leaves (unit u of the head: positions u*b .. u*b+b-1).
// The records of all heads are cut into contiguous ranges, one per warp.  Each
// record is fetched with one bulk copy into the warp's ring; the estimate is
// added to the step's anchored histogram (s >= 1).

struct __align__(16) ScoreSmem {
  unsigned char ring[kRingBytes];
  long long pref[kMaxHeads + 1];
  float anchor[kMaxHeads];
  unsigned long long red64[kDecWarps];
  unsigned long long mbar[kDecWarps][kMaxSlots];
};

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads, 1) score_kernel(const __grid_constant__ DecodeArgs a, int s) {
  pdl_wait_and_release();
  constexpr int EPC = 16 / sizeof(T);
  constexpr bool kMma = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ScoreSmem& sp = *reinterpret_cast<ScoreSmem*>(smem_raw);
  const Ctx<T, D> c(a);
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nh = a.nheads, b = a.t.block, R = a.t.refs;
  const int par = s & 1;
  const bool fp4 = kMma && a.t.planes == ZHA_PLANES_FP4;  // the routing steps read the FP4 router records
  const int rec_bytes = int(fp4 ? a.t.rec4_bytes : a.t.rec_bytes);
  // nslot record slots per warp; warps past score_warps (only when a record is
  // larger than a warp's share of the ring) do not score
  const int nslot = max(1, min(kMaxSlots, (kRingBytes / kDecWarps) / rec_bytes));
  const int score_warps = min(kDecWarps, kRingBytes / (nslot * rec_bytes));
  unsigned char* ring = sp.ring + size_t(wid) * nslot * rec_bytes;
  if (lane == 0) {
    for (int k = 0; k < nslot; ++k) mbar_init(&sp.mbar[wid][k], 1);
    mbar_init_fence();
  }
  __syncwarp();
  // ring cursors: slot of the next copy / the next record to consume, and the
  // mbarrier phase parity of the latter (flips each time it wraps)
  int slot_i = 0, slot_d = 0, in_flight = 0;
  unsigned phase_d = 0;
  float qs[EPC];
  uint32_t qf[D / 16][2];
  int qhead = -1;
  bool failed = false;  // a copy never landed: this warp stops scoring
  const long long gwarp = wid < score_warps ? (long long)blockIdx.x * score_warps + wid : -1;
  const long long nwarps = (long long)gridDim.x * score_warps;
  // ---------------- records = the roots (s = 0) or the b children of each kept
  // non-leaf of step s-1; the records of all heads are cut into contiguous
  // per-warp ranges (a small step gives most warps one record or none)
  for (int i = tid; i < nh; i += kDecThreads) {
    sp.pref[1 + i] = s == 0 ? (long long)a.n_roots : min64(max64(__ldcg(&c.hstate(i)->units), 0), a.cap_sel) * b;
    sp.anchor[i] = s == 0 ? 0.f : __ldcg(&c.hstate(i)->anchor);
  }
  __syncthreads();
  const long long total = build_prefix<kDecThreads>(sp.pref, sp.red64, nh);
  const long long u0 = gwarp < 0 ? 0 : total * gwarp / nwarps;
  const long long u1 = gwarp < 0 ? 0 : total * (gwarp + 1) / nwarps;
  for (long long ub = u0; ub < u1; ub += 32) {
    // one record per lane: its head, its position in the head's step buffer
    // (child c of unit u at u*b + c), its node code
    const long long u = ub + lane;
    int uh = 0;
    long long upos = 0;
    uint32_t ucode = 0;
    bool has = false;
    if (u < u1) {
      uh = owner_of(sp.pref, nh, u);
      const long long k = u - sp.pref[uh];
      upos = k;
      if (s == 0) {
        ucode = root_code(a, k);
        has = valid_code(a, ucode);
      } else {
        const long long unit = k / b;
        const uint32_t pc = __ldcg(c.units(uh) + unit);
        if (valid_code(a, pc) && code_level(pc) >= 2) {
          ucode = node_code(code_level(pc) - 1, code_index(pc) * uint32_t(b) + uint32_t(k - unit * b));
          has = true;
        }
      }
    }
    const unsigned mhas = __ballot_sync(0xffffffffu, has);
    if (!mhas) continue;
    constexpr int per = 1;  // records per lane
    const int items = __popc(mhas);
    // item k: the record of the k-th lane with one
    struct Cursor {
      unsigned rem;
      int child;
    };
    struct Item {
      int h;
      int src;  // the lane holding the record
      uint32_t code;
    };
    auto next_item = [&](Cursor& cur) -> Item {  // the whole warp calls it, in item order
      const int pl = __ffs(cur.rem) - 1;
      Item it;
      it.h = __shfl_sync(0xffffffffu, uh, pl);
      it.src = pl;
      it.code = __shfl_sync(0xffffffffu, ucode, pl);
      if (++cur.child == per) {
        cur.child = 0;
        cur.rem &= cur.rem - 1u;
      }
      return it;
    };
    Cursor cur_i{mhas, 0};
    Item slot_item[kMaxSlots];
    int issued = 0, done = 0;
    float my_e = -INFINITY;  // the estimate of this lane's record
    while (done < items) {
      while (issued < items && issued - done < nslot) {
        const Item it = next_item(cur_i);
        const int sl = slot_i;
        slot_i = slot_i + 1 == nslot ? 0 : slot_i + 1;
        unsigned char* slot = ring + size_t(sl) * rec_bytes;
        if (lane == 0) {
          fence_proxy_async();  // the slot's last reads (generic proxy) before the copy writes it
          const int kvh = (it.h % a.t.hq) / a.t.group;
          const int lv = code_level(it.code);
          const int64_t ix = code_index(it.code);
          bulk_load(slot, fp4 ? a.t.rec4(lv, kvh, ix) : a.t.rec(lv, kvh, ix), unsigned(rec_bytes), &sp.mbar[wid][sl]);
        }
#pragma unroll
        for (int k = 0; k < kMaxSlots; ++k)
          if (k == issued - done) slot_item[k] = it;
        ++issued;
        ++in_flight;
      }
      const int sl = slot_d;
      const unsigned parity = phase_d;
      {
        // bounded wait; on running out: report, wait for the copies in flight
        // (they read valid node records, so they land within microseconds; the
        // second bound, far above that, only guarantees termination), and stop
        // this warp
        long long it = 0;
        bool out = false;
        while (true) {
          if (it >= a.spin_limit) {
            out = true;
            break;
          }
          if (mbar_try_wait(&sp.mbar[wid][sl], parity)) break;
          ++it;
        }
        if (__any_sync(0xffffffffu, out)) {
          if (lane == 0) raise_status(a.t.status, ZHA_ERR_TIMEOUT);
          int ks = slot_d;
          unsigned kp = phase_d;
          for (int k = 0; k < in_flight; ++k) {
            for (long long d = 0; d < kDrainLimit && !mbar_try_wait(&sp.mbar[wid][ks], kp); ++d) {
            }
            if (++ks == nslot) {
              ks = 0;
              kp ^= 1u;
            }
          }
          failed = true;
          break;
        }
      }
      __syncwarp();
      const Item it = slot_item[0];
#pragma unroll
      for (int k = 0; k + 1 < kMaxSlots; ++k) slot_item[k] = slot_item[k + 1];
      if (it.h != qhead) {
        if constexpr (kMma) {
          const __nv_bfloat16* qh = static_cast<const __nv_bfloat16*>(a.Q) + size_t(it.h) * D;
          if (fp4) q_fragments_f16<D>(qh, qf, lane);
          else q_fragments<D>(qh, qf, lane);
        } else {
          c.q_slice(it.h, qs);
        }
        qhead = it.h;
      }
      const unsigned char* rec = ring + size_t(sl) * rec_bytes;
      float e;
      if constexpr (kMma) e = fp4 ? score_record_fp4<D>(rec, R, a.t.inv_sqrt_d, qf, lane)
                                  : score_record_mma<D>(rec, R, a.t.inv_sqrt_d, qf, lane);
      else e = score_record_smem<T, D>(rec, R, a.t.inv_sqrt_d, qs, lane);
      if (lane == it.src) my_e = e;
      __syncwarp();
      ++done;
      --in_flight;
      if (++slot_d == nslot) {
        slot_d = 0;
        phase_d ^= 1u;
      }
    }
    if (failed) break;
    // the batch's entries, one per lane and all lanes at once: (key, code) at
    // the entry's position, its mass in the head's anchored histogram
    const uint32_t key = has ? desc_key(my_e) : 0xffffffffu;
    if (has) {
      c.keysP(uh, par)[upos] = key;
      c.codesP(uh, par)[upos] = ucode;
      if (s >= 1) {
        unsigned long long w;
        float t;
        const int bin = anchored_bin(sp.anchor[uh], key, &w, &t);
        if (bin < 0) atomicOr(&c.hstate(uh)->ovf[par], 1);
        else atomicAdd(c.histP(uh, par) + bin, w);
      }
    }
    // the step's smallest key per head (the batch's lanes hold runs of heads;
    // usually one head)
    const int h0 = __shfl_sync(0xffffffffu, uh, __ffs(mhas) - 1);
    if (__all_sync(0xffffffffu, !has || uh == h0)) {
      const uint32_t km = __reduce_min_sync(0xffffffffu, key);
      if (lane == 0) atomicMax(&c.hstate(h0)->kinv[par], ~km);
    } else if (has) {
      atomicMax(&c.hstate(uh)->kinv[par], ~key);
    }
  }
}

// ---------------------------------------------------------------- attention
// Attended keys of head h: its kept blocks, the sink (token 0) unless block 0
// is kept, the tail after the last complete block.
template <typename T, int D>
__device__ __forceinline__ long long att_head_keys(const Ctx<T, D>& c, int h, long long* nl, bool* sink) {
  const DecodeArgs& a = c.a;
  const long long n1 = a.nl[1];
  const long long tail = a.n_tokens - n1 * a.t.block;
  *nl = 0;
  int l0 = 0;
  if (a.n_steps > 0 && a.n_roots > 0) {
    *nl = min64(max64(__ldcg(&c.hstate(h)->n_leaf), 0), a.cap_list);
    l0 = __ldcg(&c.hstate(h)->leaf0);
  }
  *sink = (n1 > 0) && !l0;
  return *nl * a.t.block + (*sink ? 1 : 0) + tail;
}

// The chunk partition of all heads' attended keys over `grid` CTAs: chunk size (>= 32 keys, so that a CTA
// owns at most about kAttItems chunks), and per-head chunk prefix in pref[0..nh].
// Each head's attended-key count, kept-leaf count and sink flag are read once
// and kept in hkeys / hnl / hsink for the chunk loop.
template <typename T, int D, int NT>
__device__ __forceinline__ void att_partition(const Ctx<T, D>& c, long long* pref, unsigned long long* red64,
                                              long long* hkeys, int* hnl, unsigned char* hsink, int grid,
                                              long long* chunk_out, long long* total_out) {
  const int nh = c.nh;
  for (int i = threadIdx.x; i < nh; i += NT) {
    long long nl;
    bool sink;
    const long long k = att_head_keys<T, D>(c, i, &nl, &sink);
    hkeys[i] = k;
    hnl[i] = int(nl);
    hsink[i] = sink ? 1 : 0;
    pref[1 + i] = k;
  }
  __syncthreads();
  const long long total_keys = build_prefix<NT>(pref, red64, nh);
  long long chunk = (total_keys + (long long)grid * kAttItems - 1) / ((long long)grid * kAttItems);
  chunk = max64(32, chunk);
  for (int i = threadIdx.x; i < nh; i += NT) pref[1 + i] = (hkeys[i] + chunk - 1) / chunk;
  __syncthreads();
  *total_out = build_prefix<NT>(pref, red64, nh);
  *chunk_out = chunk;
}

// Every head's attended keys (kept blocks, sink, tail) are cut into chunks of
// >= 32 keys; CTAs own contiguous ranges of chunks, each warp runs a chunk at a
// time (batches of keys: scores first, then one rescale of the running sums),
// and each CTA merges its chunks per head into one partial.
constexpr int kAttSlots = kAttItems + 16;  // partial slots of a CTA (per-head rounding adds up to one per head)
// The attention CTAs' partition of the chunks, written by CTA 0 after the
// items of the partial slots: [0] the chunk count, [1] the attention grid,
// [2 + h] the first chunk of head h (h = 0 .. nheads).
__device__ __forceinline__ long long* att_meta(const DecodeArgs& a, int D) {
  return reinterpret_cast<long long*>(a.attn_part + size_t(kMaxAttGrid) * kAttSlots * (2 + D));
}

struct __align__(16) AttSmem {
  float part[kAttSlots][2 + 128];
  long long pref[kMaxHeads + 1];
  long long hkeys[kMaxHeads];       // attended keys per head
  unsigned long long red64[kAttWarps];
  int hnl[kMaxHeads];               // kept level-1 blocks per head
  unsigned char hsink[kMaxHeads];   // token 0 attended as the sink (leaf block 0 not kept)
};

// CTAs per SM the attention kernel is compiled for: two for the tensor-core
// (bf16) path, whose tiles need up to 128 registers, three for the fp32 path.
template <typename T>
constexpr int att_ctas_per_sm() { return std::is_same<T, __nv_bfloat16>::value ? 2 : 3; }

template <typename T, int D>
__global__ void __launch_bounds__(kAttThreads, att_ctas_per_sm<T>()) attend_kernel(const __grid_constant__ DecodeArgs a) {
  pdl_wait_and_release();
  constexpr int EPC = 16 / sizeof(T);
  constexpr int CPR = D * sizeof(T) / 16;
  constexpr int KPW = 32 / CPR;  // keys per warp pass
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AttSmem& sm = *reinterpret_cast<AttSmem*>(smem_raw);
  const Ctx<T, D> c(a);
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nh = a.nheads, b = a.t.block;
  const long long n1 = a.nl[1];
  const DivU32 divb{uint32_t(b)};  // key index -> (block, token within it); keys per head < 2^31
  long long chunk, total_items;
  att_partition<T, D, kAttThreads>(c, sm.pref, sm.red64, sm.hkeys, sm.hnl, sm.hsink, int(gridDim.x), &chunk,
                                   &total_items);
  if (blockIdx.x == 0) {  // the partition, for the combine kernel
    long long* meta = att_meta(a, D);
    for (int i = tid; i <= nh; i += kAttThreads) meta[2 + i] = sm.pref[i];
    if (tid == 0) {
      meta[0] = total_items;
      meta[1] = gridDim.x;
    }
  }
  const long long c0 = (long long)blockIdx.x * total_items / gridDim.x;
  const long long c1 = min64((long long)(blockIdx.x + 1) * total_items / gridDim.x, c0 + kAttSlots);
  if (tid == 0 && (long long)(blockIdx.x + 1) * total_items / gridDim.x > c1) raise_status(a.t.status, ZHA_ERR_CAPACITY);
  float (*part)[2 + 128] = sm.part;
  {
    const int sub = lane / CPR, cl = lane % CPR;
    constexpr int kU = 4;
    for (long long it = c0 + wid; it < c1; it += kAttWarps) {
      const int h = owner_of(sm.pref, nh, it);
      const long long ci = it - sm.pref[h];
      const int kvh = (h % a.t.hq) / a.t.group;
      const long long nl = sm.hnl[h];
      const bool sink = sm.hsink[h] != 0;
      const long long kh = sm.hkeys[h];
      const long long leaf_keys = nl * b;
      const long long k0 = ci * chunk, k1 = min64(kh, k0 + chunk);
      float qs[EPC];
      c.q_slice(h, qs);
      const T* Kh = static_cast<const T*>(a.t.K) + size_t(kvh) * a.t.capacity * D;
      const T* Vh = static_cast<const T*>(a.t.V) + size_t(kvh) * a.t.capacity * D;
      const uint32_t* lv = c.leaves(h);
      // leaf indices of the chunk's first 32 blocks, one per lane
      uint32_t r0;
      const long long lf0 = divb.div(uint32_t(k0), &r0);
      uint32_t leaf_reg = 0;
      if (lf0 + lane < nl) leaf_reg = __ldcg(lv + lf0 + lane);
      if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        // tensor-core path: 16-key tiles, S = K q^T and O^T += V^T P with
        // mma.sync m16n8k16 as in the dense kernel, q in column 0 of the B
        // operand (the other columns are zero and ignored); the fp32 sums l
        // use the unrounded weights, O^T the weights split into hi + lo bf16
        // parts (relative rounding about 2^-16 instead of 2^-8)
        constexpr int NV = D / 32, MT = D / 16, VW = D / 64;
        const int g = lane >> 2, t4 = lane & 3;
        const __nv_bfloat16* Kb = reinterpret_cast<const __nv_bfloat16*>(Kh);
        const __nv_bfloat16* Vb = reinterpret_cast<const __nv_bfloat16*>(Vh);
        uint4 qv[NV];
        {
          const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.Q) + size_t(h) * D;
#pragma unroll
          for (int v = 0; v < NV; ++v)
            qv[v] = g == 0 ? *reinterpret_cast<const uint4*>(q + 8 * t4 + 32 * v) : make_uint4(0u, 0u, 0u, 0u);
        }
        // token of attended key idx (the whole warp calls it; idx < k1)
        auto tok_of = [&](long long idx) -> long long {
          uint32_t rb;
          const long long li = divb.div(uint32_t(idx), &rb);
          const uint32_t lr = __shfl_sync(0xffffffffu, leaf_reg, int((li - lf0) & 31));
          long long tok;
          if (idx < leaf_keys) tok = int64_t((li - lf0 < 32) ? lr : __ldcg(lv + li)) * b + rb;
          else if (sink && idx == leaf_keys) tok = 0;
          else tok = n1 * b + (idx - leaf_keys - (sink ? 1 : 0));
          if (tok < 0 || tok >= a.n_tokens) {  // a corrupted leaf index: read token 0, report
            raise_status(a.t.status, ZHA_ERR_CAPACITY);
            tok = 0;
          }
          return tok;
        };
        float om[MT][4];
#pragma unroll
        for (int i = 0; i < MT; ++i) om[i][0] = om[i][1] = om[i][2] = om[i][3] = 0.f;
        float mr[2] = {-INFINITY, -INFINITY}, lr2[2] = {0.f, 0.f};
        for (long long t0 = k0; t0 < k1; t0 += 16) {
          const long long last = k1 - 1;
          const long long tk0 = tok_of(min64(t0 + g, last)), tk1 = tok_of(min64(t0 + g + 8, last));
          uint4 kr0[NV], kr1[NV];
#pragma unroll
          for (int v = 0; v < NV; ++v) {
            kr0[v] = ldg_stream(Kb + size_t(tk0) * D + 8 * t4 + 32 * v);
            kr1[v] = ldg_stream(Kb + size_t(tk1) * D + 8 * t4 + 32 * v);
          }
          long long tv[4];
          tv[0] = tok_of(min64(t0 + 2 * t4, last));
          tv[1] = tok_of(min64(t0 + 2 * t4 + 1, last));
          tv[2] = tok_of(min64(t0 + 2 * t4 + 8, last));
          tv[3] = tok_of(min64(t0 + 2 * t4 + 9, last));
          uint4 vr[4][VW];
#pragma unroll
          for (int rr = 0; rr < 4; ++rr)
#pragma unroll
            for (int w = 0; w < VW; ++w) vr[rr][w] = ldg_stream(Vb + size_t(tv[rr]) * D + (D / 8) * g + 8 * w);
          float sv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < D / 16; ++j) {
            const int v = j >> 1, hf = j & 1;
            const uint32_t af[4] = {word_of(kr0[v], 2 * hf), word_of(kr1[v], 2 * hf), word_of(kr0[v], 2 * hf + 1),
                                    word_of(kr1[v], 2 * hf + 1)};
            const uint32_t bf[2] = {word_of(qv[v], 2 * hf), word_of(qv[v], 2 * hf + 1)};
            mma_bf16_16816(sv, af, bf);
          }
          const bool v0 = t0 + g < k1, v1 = t0 + g + 8 < k1;
#pragma unroll
          for (int i = 0; i < 4; ++i) sv[i] *= a.t.inv_sqrt_d;
          if (!v0) sv[0] = sv[1] = -INFINITY;
          if (!v1) sv[2] = sv[3] = -INFINITY;
          float pp[4];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {  // key t0 (row 0) is always valid: mx is finite
            float mx = fmaxf(sv[hh], sv[2 + hh]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float mn = fmaxf(mr[hh], mx);
            const float sc = expf(mr[hh] - mn);
            pp[hh] = expf(sv[hh] - mn);
            pp[2 + hh] = expf(sv[2 + hh] - mn);
            lr2[hh] = fmaf(lr2[hh], sc, pp[hh] + pp[2 + hh]);
            mr[hh] = mn;
#pragma unroll
            for (int i = 0; i < MT; ++i) {
              om[i][hh] *= sc;
              om[i][2 + hh] *= sc;
            }
          }
          // P as hi + lo bf16 parts (two products), so that its rounding stays near fp32
          float plo[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) plo[i] = pp[i] - __bfloat162float(__float2bfloat16_rn(pp[i]));
          const uint32_t pb[2] = {movmatrix_trans(pack_bf16(pp[0], pp[1])), movmatrix_trans(pack_bf16(pp[2], pp[3]))};
          const uint32_t pl[2] = {movmatrix_trans(pack_bf16(plo[0], plo[1])),
                                  movmatrix_trans(pack_bf16(plo[2], plo[3]))};
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            uint32_t af[4];
            if (D == 128) {
              const int w = i >> 1;
              const uint32_t sel = (i & 1) ? 0x7632u : 0x5410u;
              af[0] = __byte_perm(word_of(vr[0][0], w), word_of(vr[1][0], w), sel);
              af[1] = __byte_perm(word_of(vr[0][VW - 1], w), word_of(vr[1][VW - 1], w), sel);
              af[2] = __byte_perm(word_of(vr[2][0], w), word_of(vr[3][0], w), sel);
              af[3] = __byte_perm(word_of(vr[2][VW - 1], w), word_of(vr[3][VW - 1], w), sel);
            } else {
              const int w0 = i >> 1, w1 = (4 + i) >> 1;
              const uint32_t sel = (i & 1) ? 0x7632u : 0x5410u;
              af[0] = __byte_perm(word_of(vr[0][0], w0), word_of(vr[1][0], w0), sel);
              af[1] = __byte_perm(word_of(vr[0][0], w1), word_of(vr[1][0], w1), sel);
              af[2] = __byte_perm(word_of(vr[2][0], w0), word_of(vr[3][0], w0), sel);
              af[3] = __byte_perm(word_of(vr[2][0], w1), word_of(vr[3][0], w1), sel);
            }
            mma_bf16_16816(om[i], af, pb);
            mma_bf16_16816(om[i], af, pl);
          }
        }
        // column 0: l over the 8 lanes that share t4; m is already common to them
        lr2[0] += __shfl_xor_sync(0xffffffffu, lr2[0], 4);
        lr2[0] += __shfl_xor_sync(0xffffffffu, lr2[0], 8);
        lr2[0] += __shfl_xor_sync(0xffffffffu, lr2[0], 16);
        float* P = part[it - c0];
        if (lane == 0) {
          P[0] = mr[0];
          P[1] = lr2[0];
        }
        if (t4 == 0) {
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            const int dA = (D == 128) ? 16 * g + i : 8 * g + i;
            const int dB = (D == 128) ? 16 * g + 8 + i : 8 * g + 4 + i;
            P[2 + dA] = om[i][0];
            P[2 + dB] = om[i][2];
          }
        }
        continue;
      }
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
          uint32_t rb;
          const long long li = divb.div(uint32_t(idx), &rb);
          // every lane takes part in the shuffle; only leaf keys use the value
          const uint32_t lr = __shfl_sync(0xffffffffu, leaf_reg, int((li - lf0) & 31));
          if (idx < leaf_keys) {
            const uint32_t leaf = (li - lf0 < 32) ? lr : __ldcg(lv + li);
            tok = int64_t(leaf) * b + rb;
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
        // the batch's scores, independently; then one rescale of the running sums
        float sc8[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          float kx[EPC];
          float sv = 0.f;
          if (ok[u]) {
            unpack16<T>(kv[u], kx);
#pragma unroll
            for (int i = 0; i < EPC; ++i) sv = fmaf(kx[i], qs[i], sv);
          }
          sc8[u] = sv;
        }
#pragma unroll
        for (int off = CPR / 2; off > 0; off >>= 1) {
#pragma unroll
          for (int u = 0; u < kU; ++u) sc8[u] += __shfl_xor_sync(0xffffffffu, sc8[u], off);
        }
        float mb = m_run;
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          sc8[u] = ok[u] ? sc8[u] * a.t.inv_sqrt_d : -INFINITY;
          mb = fmaxf(mb, sc8[u]);
        }
        if (mb != -INFINITY) {
          const float r = expf(m_run - mb);
          l_run *= r;
#pragma unroll
          for (int i = 0; i < EPC; ++i) o[i] *= r;
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            if (!ok[u]) continue;
            const float pk = expf(sc8[u] - mb);
            l_run += pk;
            float vx[EPC];
            unpack16<T>(vv[u], vx);
#pragma unroll
            for (int i = 0; i < EPC; ++i) o[i] = fmaf(pk, vx[i], o[i]);
          }
          m_run = mb;
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
  // merge this CTA's chunks per head segment; one partial per segment, stored at
  // the global slot of the segment's first chunk
  for (long long seg = c0 + wid; seg < c1; seg += kAttWarps) {
    const int h = owner_of(sm.pref, nh, seg);
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
}

// ---------------------------------------------------------------- combine
// Partials (m, l, o[D]) are merged by rescaling to their common max:
// M = max m_j, L = sum e^(m_j - M) l_j, o = sum e^(m_j - M) o_j, in slot order
// (deterministic).  One warp; lane owns elements q*32 + lane.  cnt <= 32
// partials, slot_of(j) their slots (-1: none).
constexpr int kMergeBatch = 16;
template <int D, class SlotFn>
__device__ __forceinline__ void merge_partials(const float* part, int cnt, SlotFn slot_of, float& M, float& L,
                                               float (&acc)[(D + 31) / 32]) {
  const int lane = threadIdx.x & 31;
  constexpr int NQ = (D + 31) / 32;
  const long long sl = lane < cnt ? slot_of(lane) : -1;
  const float mj = sl >= 0 ? __ldcg(part + size_t(sl) * (2 + D)) : -INFINITY;
  const float lj = sl >= 0 ? __ldcg(part + size_t(sl) * (2 + D) + 1) : 0.f;
  M = mj;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float sc = (sl >= 0 && mj != -INFINITY) ? expf(mj - M) : 0.f;
  L = sc * lj;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
#pragma unroll
  for (int q = 0; q < NQ; ++q) acc[q] = 0.f;
  for (int t0 = 0; t0 < cnt; t0 += kMergeBatch) {  // kMergeBatch partials' loads in flight per lane
    float x[kMergeBatch][NQ], w[kMergeBatch];
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u) {
      const long long st = __shfl_sync(0xffffffffu, sl, (t0 + u) & 31);
      w[u] = __shfl_sync(0xffffffffu, sc, (t0 + u) & 31);
      const bool ok = t0 + u < cnt && st >= 0;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        x[u][q] = (ok && q * 32 + lane < D) ? __ldcg(part + size_t(st) * (2 + D) + 2 + q * 32 + lane) : 0.f;
      if (!ok) w[u] = 0.f;
    }
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u)
#pragma unroll
      for (int q = 0; q < NQ; ++q) acc[q] = fmaf(w[u], x[u][q], acc[q]);
  }
}

// Running merge of (M2, L2, acc2) into (M, L, acc) (one warp, same lanes).
template <int D>
__device__ __forceinline__ void merge_into(float& M, float& L, float (&acc)[(D + 31) / 32], float M2, float L2,
                                           const float (&acc2)[(D + 31) / 32]) {
  constexpr int NQ = (D + 31) / 32;
  const float Mn = fmaxf(M, M2);
  const float s1 = M == -INFINITY ? 0.f : expf(M - Mn), s2 = M2 == -INFINITY ? 0.f : expf(M2 - Mn);
  L = L * s1 + L2 * s2;
#pragma unroll
  for (int q = 0; q < NQ; ++q) acc[q] = acc[q] * s1 + acc2[q] * s2;
  M = Mn;
}

// One CTA per head, after the attention kernel.  The head's chunks [P0, P1)
// were spread over attention CTAs in contiguous chunk ranges (CTA cc starts at
// range_start(cc)); every CTA whose range meets them wrote one partial, at the
// slot max(P0, range_start(cc)).  Warp w merges a contiguous block of at most
// 32 of those partials (kMaxAttGrid / kCombWarps), then warp 0 merges the
// warps' results in warp order -> O, and writes the head's kept count and
// statistics.  The order of every sum is fixed (deterministic).
constexpr int kCombWarps = 16;
static_assert(kMaxAttGrid <= 32 * kCombWarps, "a warp merges at most 32 partials");
template <typename T, int D>
__global__ void __launch_bounds__(kCombWarps * 32) combine_kernel(const __grid_constant__ DecodeArgs a) {
  pdl_wait_and_release();
  constexpr int NQ = (D + 31) / 32;
  __shared__ float wres[kCombWarps][2 + D];
  const Ctx<T, D> c(a);
  const int h = blockIdx.x, lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const long long* meta = att_meta(a, D);
  const long long total_items = __ldcg(meta), grid = max64(__ldcg(meta + 1), 1);
  const long long P0 = __ldcg(meta + 2 + h), P1 = __ldcg(meta + 3 + h);
  auto range_start = [&](long long cc) { return cc >= grid ? total_items : (cc * total_items) / grid; };
  // attention CTAs holding chunk P0 and chunk P1 - 1
  auto cta_of = [&](long long item) {
    long long cc = (item * grid) / max64(total_items, 1);
    while (cc > 0 && range_start(cc) > item) --cc;
    while (cc + 1 < grid && range_start(cc + 1) <= item) ++cc;
    return cc;
  };
  const long long cfirst = P1 > P0 ? cta_of(P0) : 0, clast = P1 > P0 ? cta_of(P1 - 1) : -1;
  const int S = int(clast - cfirst + 1);  // partials of the head (<= grid)
  auto slot_of = [&](long long cc) -> long long {
    const long long s0 = max64(P0, range_start(cc)), s1 = min64(P1, range_start(cc + 1));
    return s0 < s1 ? s0 : -1;
  };
  // the head's counters, loaded now (they do not depend on the merge)
  HeadState* hs = c.hstate(h);
  long long nl = 0, scored = 0;
  int l0 = 0, steps = 0;
  if (wid == 0 && lane == 0 && a.n_steps > 0 && a.n_roots > 0) {
    nl = min64(max64(__ldcg(&hs->n_leaf), 0), a.cap_list);
    l0 = __ldcg(&hs->leaf0);
    scored = __ldcg(&hs->scored);
    steps = __ldcg(&hs->steps);
  }
  float M = -INFINITY, L = 0.f, acc[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) acc[q] = 0.f;
  {
    const int per = (S + kCombWarps - 1) / kCombWarps;  // <= 32
    const int j0 = min(S, wid * per), j1 = min(S, j0 + per);
    if (j1 > j0)
      merge_partials<D>(a.attn_part, j1 - j0, [&](int j) { return slot_of(cfirst + j0 + j); }, M, L, acc);
  }
  if (lane == 0) {
    wres[wid][0] = M;
    wres[wid][1] = L;
  }
#pragma unroll
  for (int q = 0; q < NQ; ++q)
    if (q * 32 + lane < D) wres[wid][2 + q * 32 + lane] = acc[q];
  __syncthreads();
  if (wid != 0) return;
  for (int w = 1; w < kCombWarps; ++w) {
    float acc2[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) acc2[q] = q * 32 + lane < D ? wres[w][2 + q * 32 + lane] : 0.f;
    merge_into<D>(M, L, acc, wres[w][0], wres[w][1], acc2);
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;  // (a head always attends a key; guard the empty case)
#pragma unroll
  for (int q = 0; q < NQ; ++q)
    if (q * 32 + lane < D) a.O[size_t(h) * D + q * 32 + lane] = acc[q] * inv;
  if (lane == 0) {
    const long long n1 = a.nl[1], b = a.t.block;
    const long long tail = a.n_tokens - n1 * b;
    if (a.kept_cnt) a.kept_cnt[h] = int32_t(nl);
    if (a.stats) {
      int64_t* st = a.stats + size_t(h) * ZHA_STAT_COUNT;
      st[ZHA_STAT_NODES_SCORED] = scored;
      st[ZHA_STAT_LEAVES_KEPT] = nl;
      st[ZHA_STAT_KEYS] = nl * b + ((n1 > 0 && !l0) ? 1 : 0) + tail;
      st[ZHA_STAT_STEPS] = steps;
    }
  }
}

// ---------------------------------------------------------------- multi-query first step
// Every query head starts from the same candidates, the forest roots, so the
// first routing step of many queries is one dense contraction: the slope rows
// of each root (R x d, bf16) times the queries of its KV head (d x queries) on
// the tensor cores (mma.sync m16n8k16: 16 slope rows x 8 query heads, d in
// 16-wide steps), e = max_j (b_j + q.mu_j / sqrt d) taken over the rows of the
// accumulator tiles.  One CTA per (root, KV head, block of sequences): the
// root's record is staged in shared memory once and each warp serves eight
// query heads of one sequence's GQA group at a time (one n-tile).  The entries go where
// the scoring kernel puts step 0's (root i at position i of the head's step
// buffer, with its largest estimate), so the select of step 0 and the later
// steps run unchanged.  bf16 configurations.
constexpr int kRootWarps = 8;
template <int D>
__global__ void __launch_bounds__(kRootWarps * 32) root_gemm_kernel(const __grid_constant__ DecodeArgs a) {
  pdl_wait_and_release();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int root = blockIdx.x, kvh = blockIdx.y;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, g = lane >> 2, t4 = lane & 3;
  const int R = a.t.refs, hq = a.t.hq, G = a.t.group;
  const int B = a.nheads / hq;
  const Ctx<__nv_bfloat16, D> c(a);
  const uint32_t code = root_code(a, root);
  if (!valid_code(a, code)) return;
  // the root's record: R slope rows of D bf16, then R fp32 intercepts
  const unsigned char* rec = reinterpret_cast<const unsigned char*>(a.t.rec(code_level(code), kvh, code_index(code)));
  const int rec_words = int(a.t.rec_bytes / 16);
  for (int i = threadIdx.x; i < rec_words; i += blockDim.x)
    reinterpret_cast<uint4*>(smem_raw)[i] = *reinterpret_cast<const uint4*>(rec + size_t(i) * 16);
  __syncthreads();
  const __nv_bfloat16* mu = reinterpret_cast<const __nv_bfloat16*>(smem_raw);
  const float* bias = reinterpret_cast<const float*>(smem_raw + size_t(R) * D * 2);
  const int ntiles = (G + 7) / 8;
  for (int item = blockIdx.z * kRootWarps + wid; item < B * ntiles; item += gridDim.z * kRootWarps) {
    const int bb = item / ntiles, n0 = (item - bb * ntiles) * 8;
    // query head of column g of this n-tile: head n0 + g of the KV head's group in sequence bb (columns past
    // the group read its last head; their results are dropped)
    const int hcol = bb * hq + kvh * G + min(n0 + g, G - 1);
    const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(a.Q) + size_t(hcol) * D + 2 * t4;
    float best0 = -INFINITY, best1 = -INFINITY;  // columns 2 t4 and 2 t4 + 1
    for (int m0 = 0; m0 < R; m0 += 16) {
      const int r0 = min(m0 + g, R - 1), r1 = min(m0 + g + 8, R - 1);
      const __nv_bfloat16* a0p = mu + size_t(r0) * D + 2 * t4;
      const __nv_bfloat16* a1p = mu + size_t(r1) * D + 2 * t4;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k0 = 0; k0 < D; k0 += 16) {
        const uint32_t af[4] = {*reinterpret_cast<const uint32_t*>(a0p + k0), *reinterpret_cast<const uint32_t*>(a1p + k0),
                                *reinterpret_cast<const uint32_t*>(a0p + k0 + 8),
                                *reinterpret_cast<const uint32_t*>(a1p + k0 + 8)};
        const uint32_t bf[2] = {*reinterpret_cast<const uint32_t*>(qp + k0), *reinterpret_cast<const uint32_t*>(qp + k0 + 8)};
        mma_bf16_16816(acc, af, bf);
      }
      // rows m0 + g and m0 + g + 8 of columns 2 t4, 2 t4 + 1
      const int j0 = m0 + g, j1 = m0 + g + 8;
      if (j0 < R) {
        best0 = fmaxf(best0, fmaf(acc[0], a.t.inv_sqrt_d, bias[j0]));
        best1 = fmaxf(best1, fmaf(acc[1], a.t.inv_sqrt_d, bias[j0]));
      }
      if (j1 < R) {
        best0 = fmaxf(best0, fmaf(acc[2], a.t.inv_sqrt_d, bias[j1]));
        best1 = fmaxf(best1, fmaf(acc[3], a.t.inv_sqrt_d, bias[j1]));
      }
    }
    // the maximum over the rows: lanes with the same t4 (xor over g)
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      best0 = fmaxf(best0, __shfl_xor_sync(0xffffffffu, best0, off));
      best1 = fmaxf(best1, __shfl_xor_sync(0xffffffffu, best1, off));
    }
    if (g == 0) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int col = n0 + 2 * t4 + u;
        if (col >= G) continue;
        const int h = bb * hq + kvh * G + col;
        const uint32_t key = desc_key(u == 0 ? best0 : best1);
        c.keysP(h, 0)[root] = key;
        c.codesP(h, 0)[root] = code;
        atomicMax(&c.hstate(h)->kinv[0], ~key);
      }
    }
  }
}

// ------------------------------------------------------------------ host launcher
static int device_sms() {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// Launch with programmatic stream serialization (see pdl_wait_and_release).
template <typename... Args>
static void launch_pdl(void (*kern)(Args...), dim3 grid, unsigned block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kern, args...);
}

// The large dynamic shared memory of the decode kernels is an attribute of each
// kernel on each device: set once per (kernel instance, device), under a lock.
template <typename T, int D>
static cudaError_t configure_decode_t() {
  static std::mutex mu;
  static bool done[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(score_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sizeof(ScoreSmem)));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(select_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sizeof(DecSmem)));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attend_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sizeof(AttSmem)));
  if (e != cudaSuccess) return e;
  done[dev] = true;
  return cudaSuccess;
}

template <typename T, int D>
static cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t st) {
  {
    const cudaError_t e = configure_decode_t<T, D>();
    if (e != cudaSuccess) return e;
  }
  const int sms = device_sms();
  const unsigned nh = unsigned(a.nheads);
  const bool routed = a.n_steps > 0 && a.n_roots > 0;
  int launches = 0;
  if (routed) {
    for (int s = 0; s < a.n_steps; ++s) {
      if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        if (s == 0 && a.root_gemm) {  // the shared first step as one tensor-core contraction
          const int items = (a.nheads / a.t.hq) * ((a.t.group + 7) / 8);
          const unsigned zb = unsigned((items + 8 * kRootWarps - 1) / (8 * kRootWarps));
          launch_pdl(root_gemm_kernel<D>, dim3(unsigned(a.n_roots), unsigned(a.t.hkv), zb), kRootWarps * 32,
                     size_t(a.t.rec_bytes), st, a);
          launch_pdl(select_kernel<T, D>, nh, kDecThreads, sizeof(DecSmem), st, a, s);
          launches += 2;
          continue;
        }
      }
      launch_pdl(score_kernel<T, D>, unsigned(sms), kDecThreads, sizeof(ScoreSmem), st, a, s);
      launch_pdl(select_kernel<T, D>, nh, kDecThreads, sizeof(DecSmem), st, a, s);
      launches += 2;
    }
  }
  const int att_grid = min(kMaxAttGrid, att_ctas_per_sm<T>() * sms);  // one wave
  launch_pdl(attend_kernel<T, D>, unsigned(att_grid), kAttThreads, sizeof(AttSmem), st, a);
  launch_pdl(combine_kernel<T, D>, nh, kCombWarps * 32, 0, st, a);
  launches += 2;
  count_launches(launches);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, int dtype, cudaStream_t st) {
  if (dtype == ZHA_BF16)
    return a.t.d == 128 ? launch_decode_t<__nv_bfloat16, 128>(a, st) : launch_decode_t<__nv_bfloat16, 64>(a, st);
  return a.t.d == 128 ? launch_decode_t<float, 128>(a, st) : launch_decode_t<float, 64>(a, st);
}

// Head states and leaf bitmaps, one region cleared together.
size_t decode_flow_bytes(int nheads, int64_t cap_sel) {
  return size_t(nheads) * (sizeof(HeadState) + size_t(decode_bitmap_words(cap_sel)) * 4);
}
// Per-head routing workspace: step keys and codes in two parity buffers, two
// anchored histograms, the units of the next scoring phase, the kept leaves.
uint64_t decode_ws_bytes(int64_t cap_sel, int64_t cap_list) {
  const uint64_t cap4 = (uint64_t(cap_sel) + 3) & ~uint64_t(3);
  return cap4 * 20 + 2 * kBins * 8 + uint64_t(cap_list) * 4;
}
int decode_max_heads() { return kMaxHeads; }
// attention partial slots of one call: at most kAttItems per CTA, one more per head
uint64_t decode_part_items(int nheads) { return uint64_t(kMaxAttGrid) * (kAttItems + 16) + uint64_t(nheads) + 64; }

}  // namespace zha
