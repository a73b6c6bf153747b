// Dense decode attention (the comparator the tree is measured against):
// o = softmax(q.K^T / sqrt(d)) V over every cached token.
//
// Split-KV flash decode.  The key range of each (sequence, KV head) is split
// into `splits` contiguous ranges, one CTA each; a CTA keeps an online softmax
// (running max, running sum, running output) per query head and writes one
// partial per head.  A second kernel (one CTA per query head and sequence)
// combines the partials.
//
// bf16 path: one CTA serves the whole GQA group (<= 8 query heads) so every
// K/V byte is read once for all of them.  Per 16-key tile a warp computes
// S^T = K Q^T with mma.sync m16n8k16 (keys x heads) and O^T += V^T P with the
// same instruction (head dim x heads), P moved from the accumulator layout to
// the operand layout with movmatrix and split into hi + lo bf16 parts (two
// products, so the weights keep about 16 bits instead of 8).  K and V are loaded straight from global
// memory into registers with 16-byte loads; the head dimension is permuted
// consistently between the operands so that every fragment is whole 32-bit
// words of those loads.  The work is HBM-bound (about 4 flop per byte at 8
// heads), so the tensor core is used only to keep the FMA pipe from becoming
// the limit.
// fp32 path: one CTA per query head, CUDA cores.
#include <mutex>

#include "zha_args.cuh"

namespace zha {

constexpr int kDenseThreads = 128;
constexpr int kDenseWarps = kDenseThreads / 32;
constexpr int kDenseTile = 16;

// Combine the split partials of one query head: one CTA per (head, sequence).
// o = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s with M = max_s m_s.
template <int D>
__global__ void __launch_bounds__(256) dense_combine_kernel(DenseArgs a) {
  constexpr int NP = 256 / D;  // threads per output element
  const int h = blockIdx.x, bb = blockIdx.y, tid = threadIdx.x;
  const float* P = a.part + (size_t(bb) * a.hq + h) * a.splits * (D + 2);
  extern __shared__ float csm[];  // scale[splits], then red[NP][D]
  float* scale = csm;
  float* red = csm + a.splits;
  __shared__ float wred[8];
  float m = -INFINITY;
  for (int s = tid; s < a.splits; s += blockDim.x) m = fmaxf(m, __ldcg(P + size_t(s) * (D + 2)));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((tid & 31) == 0) wred[tid >> 5] = m;
  __syncthreads();
  float M = -INFINITY;
  for (int w = 0; w < 8; ++w) M = fmaxf(M, wred[w]);
  __syncthreads();
  float l = 0.f;
  for (int s = tid; s < a.splits; s += blockDim.x) {
    const float ms = __ldcg(P + size_t(s) * (D + 2));
    const float sc = ms == -INFINITY ? 0.f : expf(ms - M);
    scale[s] = sc;
    l = fmaf(sc, __ldcg(P + size_t(s) * (D + 2) + 1), l);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  if ((tid & 31) == 0) wred[tid >> 5] = l;
  __syncthreads();
  float L = 0.f;
  for (int w = 0; w < 8; ++w) L += wred[w];
  const int e = tid % D, part = tid / D;
  float acc = 0.f;
  for (int s = part; s < a.splits; s += NP) acc = fmaf(scale[s], __ldcg(P + size_t(s) * (D + 2) + 2 + e), acc);
  red[part * D + e] = acc;
  __syncthreads();
  if (part == 0) {
    for (int q = 1; q < NP; ++q) acc += red[q * D + e];
    a.O[(size_t(bb) * a.hq + h) * D + e] = acc / L;
  }
}

// ------------------------------------------------------------------ bf16, tensor-core path
template <int D>
__global__ void __launch_bounds__(kDenseThreads, 4) dense_mma_kernel(DenseArgs a) {
  constexpr int NV = D / 32;  // 16-byte Q/K vectors per thread per row
  constexpr int MT = D / 16;  // m-tiles of O^T
  const int split = blockIdx.x, kvh = blockIdx.y, bb = blockIdx.z;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int64_t k_begin = int64_t(split) * a.per;
  const int64_t k_end = min64(a.n, k_begin + a.per);
  const __nv_bfloat16* Kh = static_cast<const __nv_bfloat16*>(a.K) + size_t(kvh) * a.ld * D;
  const __nv_bfloat16* Vh = static_cast<const __nv_bfloat16*>(a.V) + size_t(kvh) * a.ld * D;

  // Q fragment (B operand): head g, elements 8*t4 + 32*v + [0, 8)
  uint4 qv[NV];
  {
    const bool valid = g < a.group;
    const __nv_bfloat16* q =
        static_cast<const __nv_bfloat16*>(a.Q) + (size_t(bb) * a.hq + kvh * a.group + (valid ? g : 0)) * D;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      qv[v] = valid ? *reinterpret_cast<const uint4*>(q + 8 * t4 + 32 * v) : make_uint4(0, 0, 0, 0);
    }
  }
  float o[MT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

  for (int64_t t0 = k_begin + int64_t(wid) * kDenseTile; t0 < k_end; t0 += int64_t(kDenseWarps) * kDenseTile) {
    const int64_t last = k_end - 1;
    // K rows g and g+8 of the tile
    const int64_t kr0 = min64(t0 + g, last), kr1 = min64(t0 + g + 8, last);
    uint4 k0[NV], k1[NV];
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      k0[v] = ldg_stream(Kh + size_t(kr0) * D + 8 * t4 + 32 * v);
      k1[v] = ldg_stream(Kh + size_t(kr1) * D + 8 * t4 + 32 * v);
    }
    // V rows 2t4, 2t4+1, 2t4+8, 2t4+9, elements of this thread's d-range
    constexpr int VW = D / 64;  // 16-byte vectors per V row per thread (2 for D=128, 1 for D=64)
    uint4 vr[4][VW];
    {
      const int64_t rows[4] = {min64(t0 + 2 * t4, last), min64(t0 + 2 * t4 + 1, last),
                               min64(t0 + 2 * t4 + 8, last), min64(t0 + 2 * t4 + 9, last)};
#pragma unroll
      for (int rr = 0; rr < 4; ++rr)
#pragma unroll
        for (int w = 0; w < VW; ++w) vr[rr][w] = ldg_stream(Vh + size_t(rows[rr]) * D + (D / 8) * g + 8 * w);
    }
    // S^T = K Q^T  (16 keys x 8 heads)
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < D / 16; ++j) {
      const int v = j >> 1, hf = j & 1;
      const uint32_t af[4] = {word_of(k0[v], 2 * hf), word_of(k1[v], 2 * hf), word_of(k0[v], 2 * hf + 1),
                              word_of(k1[v], 2 * hf + 1)};
      const uint32_t bf[2] = {word_of(qv[v], 2 * hf), word_of(qv[v], 2 * hf + 1)};
      mma_bf16_16816(s, af, bf);
    }
    // keys g (s[0], s[1]) and g+8 (s[2], s[3]); heads 2t4 (s[0], s[2]) and 2t4+1 (s[1], s[3])
    const bool v0 = t0 + g < k_end, v1 = t0 + g + 8 < k_end;
#pragma unroll
    for (int i = 0; i < 4; ++i) s[i] *= a.inv_sqrt_d;
    if (!v0) s[0] = s[1] = -INFINITY;
    if (!v1) s[2] = s[3] = -INFINITY;
    float p[4];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float mx = fmaxf(s[hh], s[2 + hh]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float mn = fmaxf(m_run[hh], mx);
      const float sc = expf(m_run[hh] - mn);
      p[hh] = expf(s[hh] - mn);
      p[2 + hh] = expf(s[2 + hh] - mn);
      l_run[hh] = fmaf(l_run[hh], sc, p[hh] + p[2 + hh]);
      m_run[hh] = mn;
#pragma unroll
      for (int i = 0; i < MT; ++i) {
        o[i][hh] *= sc;
        o[i][2 + hh] *= sc;
      }
    }
    // P (keys x heads) -> B operand (keys x heads, column-major) via transpose, as hi + lo bf16 parts
    // (two products), so that the rounding of the weights stays near fp32 instead of 2^-8
    float plo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) plo[i] = p[i] - __bfloat162float(__float2bfloat16_rn(p[i]));
    const uint32_t pb[2] = {movmatrix_trans(pack_bf16(p[0], p[1])), movmatrix_trans(pack_bf16(p[2], p[3]))};
    const uint32_t pl[2] = {movmatrix_trans(pack_bf16(plo[0], plo[1])), movmatrix_trans(pack_bf16(plo[2], plo[3]))};
    // O^T += V^T P
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      // d rows of m-tile i for this thread: row g -> element i of the thread's
      // range, row g+8 -> element MT/2... (see header comment)
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
      mma_bf16_16816(o[i], af, pb);
      mma_bf16_16816(o[i], af, pl);
    }
  }
  // reduce l over the 8 lanes that share t4
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 4);
    l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 8);
    l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 16);
  }
  // combine the warps of the CTA in shared memory: per head m, l, o[D]
  __shared__ float wm[kDenseWarps][8], wl[kDenseWarps][8];
  __shared__ float wo[kDenseWarps][8][D];
  if (g == 0) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      wm[wid][2 * t4 + hh] = m_run[hh];
      wl[wid][2 * t4 + hh] = l_run[hh];
    }
  }
#pragma unroll
  for (int i = 0; i < MT; ++i) {
    const int dA = (D == 128) ? 16 * g + i : 8 * g + i;
    const int dB = (D == 128) ? 16 * g + 8 + i : 8 * g + 4 + i;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      wo[wid][2 * t4 + hh][dA] = o[i][hh];
      wo[wid][2 * t4 + hh][dB] = o[i][2 + hh];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < a.group * (D + 2); idx += blockDim.x) {
    const int hh = idx / (D + 2), e = idx % (D + 2);
    float M = -INFINITY;
    for (int w = 0; w < kDenseWarps; ++w) M = fmaxf(M, wm[w][hh]);
    float val;
    if (e == 0) {
      val = M;
    } else {
      val = 0.f;
      for (int w = 0; w < kDenseWarps; ++w) {
        if (wm[w][hh] == -INFINITY) continue;
        val = fmaf(expf(wm[w][hh] - M), e == 1 ? wl[w][hh] : wo[w][hh][e - 2], val);
      }
    }
    a.part[((size_t(bb) * a.hq + kvh * a.group + hh) * a.splits + split) * (D + 2) + e] = val;
  }
}

// ------------------------------------------------------------------ CUDA-core path (fp32, any group)
template <typename T, int D>
__global__ void __launch_bounds__(256) dense_scalar_kernel(DenseArgs a) {
  constexpr int EPC = 16 / sizeof(T);
  constexpr int CPR = D * sizeof(T) / 16;
  constexpr int KPW = 32 / CPR;
  constexpr int W = 8;
  const int split = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
  const int kvh = h / a.group;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int sub = lane / CPR, cl = lane % CPR;
  const int64_t k_begin = int64_t(split) * a.per, k_end = min64(a.n, k_begin + a.per);
  const T* Kh = static_cast<const T*>(a.K) + size_t(kvh) * a.ld * D;
  const T* Vh = static_cast<const T*>(a.V) + size_t(kvh) * a.ld * D;
  float qs[EPC];
  unpack16<T>(*reinterpret_cast<const uint4*>(static_cast<const T*>(a.Q) + (size_t(bb) * a.hq + h) * D + cl * EPC),
              qs);
  float m_run = -INFINITY, l_run = 0.f, o[EPC];
#pragma unroll
  for (int i = 0; i < EPC; ++i) o[i] = 0.f;
  for (int64_t wb = k_begin + int64_t(wid) * KPW; wb < k_end; wb += int64_t(W) * KPW) {
    const int64_t k = wb + sub;
    const bool ok = k < k_end;
    const int64_t kk = ok ? k : k_end - 1;
    float kx[EPC], vx[EPC];
    unpack16<T>(ldg_stream(Kh + size_t(kk) * D + cl * EPC), kx);
    unpack16<T>(ldg_stream(Vh + size_t(kk) * D + cl * EPC), vx);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < EPC; ++i) s = fmaf(kx[i], qs[i], s);
#pragma unroll
    for (int off = CPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (ok) {
      s *= a.inv_sqrt_d;
      const float mn = fmaxf(m_run, s);
      const float sc = expf(m_run - mn), pk = expf(s - mn);
      l_run = fmaf(l_run, sc, pk);
#pragma unroll
      for (int i = 0; i < EPC; ++i) o[i] = fmaf(pk, vx[i], o[i] * sc);
      m_run = mn;
    }
  }
  __shared__ float gm[W * KPW], gl[W * KPW], go[W * KPW][D];
  const int grp = wid * KPW + sub;
  if (cl == 0) {
    gm[grp] = m_run;
    gl[grp] = l_run;
  }
#pragma unroll
  for (int i = 0; i < EPC; ++i) go[grp][cl * EPC + i] = o[i];
  __syncthreads();
  for (int e = threadIdx.x; e < D + 2; e += blockDim.x) {
    float M = -INFINITY;
    for (int gi = 0; gi < W * KPW; ++gi) M = fmaxf(M, gm[gi]);
    float val = 0.f;
    if (e == 0) {
      val = M;
    } else {
      for (int gi = 0; gi < W * KPW; ++gi) {
        if (gm[gi] == -INFINITY) continue;
        val = fmaf(expf(gm[gi] - M), e == 1 ? gl[gi] : go[gi][e - 2], val);
      }
    }
    a.part[((size_t(bb) * a.hq + h) * a.splits + split) * (D + 2) + e] = val;
  }
}

// ------------------------------------------------------------------ fixed scratch
// Split partials of zha_dense_decode_noalloc live in this array instead of
// caller memory: 2^20 floats (4 MiB) on every device that loads the library,
// held until the process exits.  Every call writes the partials it later
// reads, so nothing in it has to start at zero.
constexpr size_t kDenseStaticFloats = size_t(1) << 20;
static __device__ __align__(256) float g_dense_static_part[kDenseStaticFloats];

size_t dense_static_floats() { return kDenseStaticFloats; }

// Device address of the array on the current device.  A host-side reference
// to g_dense_static_part is only a stand-in, so the address is looked up once
// per device (with that device current) and cached.
cudaError_t dense_static_scratch(float** out) {
  static std::mutex mu;
  static float* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dense_static_part);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<float*>(p);
  }
  *out = addr[dev];
  return cudaSuccess;
}

// ------------------------------------------------------------------ host side
int dense_target_splits() { return 148 * 4; }  // four CTAs per SM of a B200

void dense_plan(int B, int hkv, int64_t n, int* splits, int64_t* per) {
  const int target = dense_target_splits();
  int64_t s = (target + int64_t(B) * hkv - 1) / (int64_t(B) * hkv);
  const int64_t max_s = (n + 63) / 64;
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  int64_t p = (n + s - 1) / s;
  p = (p + 63) / 64 * 64;
  if (p < 64) p = 64;
  *per = p;
  *splits = int((n + p - 1) / p);
  if (*splits < 1) *splits = 1;
}

bool dense_uses_mma(int dtype, int group) { return dtype == ZHA_BF16 && group <= 8; }

cudaError_t launch_dense(const DenseArgs& a0, int dtype, int d, int B, cudaStream_t st) {
  DenseArgs a = a0;
  count_launches(2);
  if (dense_uses_mma(dtype, a.group)) {
    dim3 grid(unsigned(a.splits), unsigned(a.hkv), unsigned(B));
    if (d == 128) dense_mma_kernel<128><<<grid, kDenseThreads, 0, st>>>(a);
    else dense_mma_kernel<64><<<grid, kDenseThreads, 0, st>>>(a);
  } else {
    dim3 grid(unsigned(a.splits), unsigned(a.hq), unsigned(B));
    if (dtype == ZHA_BF16) {
      if (d == 128) dense_scalar_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(a);
      else dense_scalar_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(a);
    } else {
      if (d == 128) dense_scalar_kernel<float, 128><<<grid, 256, 0, st>>>(a);
      else dense_scalar_kernel<float, 64><<<grid, 256, 0, st>>>(a);
    }
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t sm = (size_t(a.splits) + 256) * sizeof(float);
  dim3 cgrid(unsigned(a.hq), unsigned(B));
  if (d == 128) dense_combine_kernel<128><<<cgrid, 256, sm, st>>>(a);
  else dense_combine_kernel<64><<<cgrid, 256, sm, st>>>(a);
  return cudaGetLastError();
}

}  // namespace zha
