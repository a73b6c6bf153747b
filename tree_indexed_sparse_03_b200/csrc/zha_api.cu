// Host side of the C ABI declared in include/zha.h: validation, buffer
// layouts, tree bookkeeping and kernel launches.  No device memory is
// allocated here; every buffer belongs to the caller.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>

#include "zha_common.cuh"

namespace zha {
// kernels (zha_build.cu, zha_decode.cu, zha_dense.cu)
cudaError_t launch_tree_update(const TreeDev& t, int dtype, int64_t n_old, int64_t n_new, cudaStream_t st);
cudaError_t launch_append_copy(const TreeDev& t, int dtype, const void* Kn, const void* Vn, int64_t n, int64_t m,
                               cudaStream_t st);
bool append_fast_ok(const TreeDev& t, int64_t n, int64_t m);
cudaError_t launch_append_fast(const TreeDev& t, int dtype, const void* Kn, const void* Vn, int64_t n, int64_t m,
                               cudaStream_t st);
size_t chunk_smem_bytes(int dtype, int d, int block, int chunk_level, int R);
size_t decode_flow_bytes(int nheads, int64_t cap_sel);
uint64_t decode_ws_bytes(int64_t cap_sel, int64_t cap_list);
int decode_max_heads();
uint64_t decode_part_items(int nheads);
void dense_plan(int B, int hkv, int64_t n, int* splits, int64_t* per);
int dense_target_splits();
size_t dense_static_floats();
cudaError_t dense_static_scratch(float** out);
}  // namespace zha

#include "zha_args.cuh"

using namespace zha;

static std::atomic<uint64_t> g_launches{0};

void zha::count_launches(int n) { g_launches.fetch_add(uint64_t(n), std::memory_order_relaxed); }

namespace {

thread_local std::string g_err;

int fail(int code, const char* msg) {
  g_err = msg;
  return code;
}

int fail_cuda(cudaError_t e, const char* where) {
  g_err = std::string(where) + ": " + cudaGetErrorString(e);
  return ZHA_ERR_CUDA;
}

struct Layout {
  int S;                                 // chunk level
  int64_t cap_nodes[kMaxLevels + 1];
  int64_t pow_b[kMaxLevels + 1];
  uint64_t rec_off[kMaxLevels + 1], f_off[kMaxLevels + 1], up_off[kMaxLevels + 1];
  uint64_t rec4_off[kMaxLevels + 1], rec4_bytes;  // FP4 router records (planes = ZHA_PLANES_FP4)
  uint64_t rec_bytes, up_bytes, node_bytes;
  // scratch
  uint64_t status_off, part_off, part_items, flow_off, flow_bytes, ws_off, ws_per_bh, stage_off, scratch_bytes;
  int64_t cap_sel, cap_list;
  uint64_t stage_k, stage_v, stage_q, stage_o;
};

uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

constexpr long long kDefaultSpinLimit = 1ll << 22;  // bound of the decode's waits on record copies (try_wait rounds)

int elem_size(int dtype) { return dtype == ZHA_BF16 ? 2 : 4; }

int validate(const zha_config* c) {
  if (!c) return fail(ZHA_ERR_INVALID, "config is NULL");
  if (c->d != 64 && c->d != 128) return fail(ZHA_ERR_UNSUPPORTED, "head dim must be 64 or 128");
  if (c->n_kv_heads < 1 || c->n_q_heads < 1) return fail(ZHA_ERR_INVALID, "head counts must be >= 1");
  if (c->n_q_heads % c->n_kv_heads) return fail(ZHA_ERR_UNSUPPORTED, "n_q_heads must be a multiple of n_kv_heads");
  if (c->block < 2) return fail(ZHA_ERR_UNSUPPORTED, "block must be >= 2");
  if (c->levels < 1 || c->levels > kMaxLevels) return fail(ZHA_ERR_UNSUPPORTED, "levels must be in [1, 20]");
  if (c->n_refs < 1 || c->n_refs > kMaxRefs) return fail(ZHA_ERR_UNSUPPORTED, "n_refs must be in [1, 32]");
  if (!(c->p > 0.f) || !(c->p <= 1.f)) return fail(ZHA_ERR_INVALID, "p must be in (0, 1]");
  if (c->dtype != ZHA_F32 && c->dtype != ZHA_BF16) return fail(ZHA_ERR_UNSUPPORTED, "dtype must be ZHA_F32 or ZHA_BF16");
  if (c->capacity < 1 || c->capacity >= (int64_t(1) << 31)) return fail(ZHA_ERR_INVALID, "capacity must be in [1, 2^31)");
  if (c->capacity / c->block >= (int64_t(1) << 27)) return fail(ZHA_ERR_UNSUPPORTED, "capacity / block must be < 2^27");
  if (c->max_batch < 1 || c->max_batch > 65535) return fail(ZHA_ERR_INVALID, "max_batch must be in [1, 65535]");
  if (c->planes != ZHA_PLANES_KEY && c->planes != ZHA_PLANES_FP4)
    return fail(ZHA_ERR_INVALID, "planes must be ZHA_PLANES_KEY or ZHA_PLANES_FP4");
  if (c->planes == ZHA_PLANES_FP4 && c->dtype != ZHA_BF16)
    return fail(ZHA_ERR_UNSUPPORTED, "FP4 router planes need a bf16 configuration");
  if (int64_t(c->max_batch) * c->n_q_heads > decode_max_heads())
    return fail(ZHA_ERR_UNSUPPORTED, "max_batch * n_q_heads must be <= 1024");
  // block^levels must fit comfortably in int64
  double span = std::pow(double(c->block), double(c->levels));
  if (span > 4e18) return fail(ZHA_ERR_UNSUPPORTED, "block^levels too large");
  return ZHA_OK;
}

int chunk_level_for(const zha_config* c) {
  int S = 1;
  int64_t w = c->block;
  while (S < c->levels && w * c->block <= 64) {
    w *= c->block;
    ++S;
  }
  return S;
}

int make_layout(const zha_config* c, Layout* L) {
  int rc = validate(c);
  if (rc) return rc;
  std::memset(L, 0, sizeof(*L));
  const int es = elem_size(c->dtype);
  L->S = chunk_level_for(c);
  if (chunk_smem_bytes(c->dtype, c->d, c->block, L->S, c->n_refs) > 200 * 1024)
    return fail(ZHA_ERR_UNSUPPORTED, "block too large for the build kernel's shared memory");
  L->rec_bytes = uint64_t(c->n_refs) * c->d * es + ((uint64_t(c->n_refs) * 4 + 15) & ~uint64_t(15));
  L->up_bytes = (uint64_t(c->n_refs) * (c->d + 2) * 4 + 15) & ~uint64_t(15);  // 16-byte rows for vector stores
  uint64_t off = 0;
  int64_t pw = 1;
  L->pow_b[0] = 1;
  L->cap_nodes[0] = c->capacity;
  for (int l = 1; l <= c->levels; ++l) {
    pw *= c->block;
    L->pow_b[l] = pw;
    L->cap_nodes[l] = c->capacity / pw;
    L->rec_off[l] = off;
    off = align256(off + uint64_t(c->n_kv_heads) * L->cap_nodes[l] * L->rec_bytes);
    L->f_off[l] = off;
    off = align256(off + uint64_t(c->n_kv_heads) * L->cap_nodes[l] * c->n_refs * 4);
  }
  for (int l = L->S; l < c->levels; ++l) {
    L->up_off[l] = off;
    off = align256(off + uint64_t(c->n_kv_heads) * L->cap_nodes[l] * L->up_bytes);
  }
  if (c->planes == ZHA_PLANES_FP4) {
    L->rec4_bytes = uint64_t(c->n_refs) * (c->d / 2 + c->d / 16) + ((uint64_t(c->n_refs) * 4 + 15) & ~uint64_t(15));
    L->rec4_bytes = (L->rec4_bytes + 15) & ~uint64_t(15);
    for (int l = 1; l <= c->levels; ++l) {
      L->rec4_off[l] = off;
      off = align256(off + uint64_t(c->n_kv_heads) * L->cap_nodes[l] * L->rec4_bytes);
    }
  }
  L->node_bytes = off > 0 ? off : 256;
  // scratch: status word, attend partials, per (sequence, query head)
  // routing state and workspace, host-step staging
  L->status_off = 0;
  const int64_t n1cap = L->cap_nodes[1] > 0 ? L->cap_nodes[1] : 1;
  L->cap_sel = n1cap;
  L->cap_list = n1cap + 64;
  const uint64_t nheads = uint64_t(c->max_batch) * c->n_q_heads;
  L->part_off = 256;
  L->part_items = decode_part_items(int(nheads));
  L->flow_off = align256(L->part_off + L->part_items * (c->d + 2) * 4);
  // head states and leaf bitmaps, cleared together
  L->flow_bytes = decode_flow_bytes(int(nheads), L->cap_sel);
  L->ws_off = align256(L->flow_off + L->flow_bytes);
  L->ws_per_bh = align256(decode_ws_bytes(L->cap_sel, L->cap_list));
  uint64_t s = L->ws_off + L->ws_per_bh * uint64_t(c->max_batch) * c->n_q_heads;
  L->stage_off = s;
  L->stage_k = s;
  s = align256(s + uint64_t(c->n_kv_heads) * c->d * es);
  L->stage_v = s;
  s = align256(s + uint64_t(c->n_kv_heads) * c->d * es);
  L->stage_q = s;
  s = align256(s + uint64_t(c->max_batch) * c->n_q_heads * c->d * es);
  L->stage_o = s;
  s = align256(s + uint64_t(c->max_batch) * c->n_q_heads * c->d * 4);
  L->scratch_bytes = s;
  return ZHA_OK;
}

}  // namespace

struct zha_tree {
  zha_config cfg;
  Layout L;
  TreeDev dev;
  char* scratch;
  int64_t n;
  int device;
  long long spin_limit;  // bound of the decode's waits on record copies
  bool flow_dirty;               // the routing flow state must be zeroed before the next decode
  float step_p[kMaxLevels];      // per-step thresholds (n_step_p of them; 0: the configuration's p)
  int n_step_p;
};

extern "C" {

const char* zha_last_error(void) { return g_err.c_str(); }

uint64_t zha_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int zha_tree_bytes(const zha_config* cfg, size_t* node_bytes, size_t* scratch_bytes) {
  Layout L;
  int rc = make_layout(cfg, &L);
  if (rc) return rc;
  if (node_bytes) *node_bytes = L.node_bytes;
  if (scratch_bytes) *scratch_bytes = L.scratch_bytes;
  return ZHA_OK;
}

int zha_tree_layout(const zha_config* cfg, int32_t level, size_t* rec_offset, size_t* f_offset, int64_t* cap_nodes,
                    size_t* rec_bytes) {
  Layout L;
  int rc = make_layout(cfg, &L);
  if (rc) return rc;
  if (level < 1 || level > cfg->levels) return fail(ZHA_ERR_INVALID, "level out of range");
  if (rec_offset) *rec_offset = L.rec_off[level];
  if (f_offset) *f_offset = L.f_off[level];
  if (cap_nodes) *cap_nodes = L.cap_nodes[level];
  if (rec_bytes) *rec_bytes = L.rec_bytes;
  return ZHA_OK;
}

int zha_tree_layout_fp4(const zha_config* cfg, int32_t level, size_t* rec_offset, size_t* rec_bytes) {
  Layout L;
  int rc = make_layout(cfg, &L);
  if (rc) return rc;
  if (cfg->planes != ZHA_PLANES_FP4) return fail(ZHA_ERR_INVALID, "the configuration has no FP4 router planes");
  if (level < 1 || level > cfg->levels) return fail(ZHA_ERR_INVALID, "level out of range");
  if (rec_offset) *rec_offset = L.rec4_off[level];
  if (rec_bytes) *rec_bytes = L.rec4_bytes;
  return ZHA_OK;
}

int zha_tree_create(const zha_config* cfg, void* K, void* V, const void* refs, void* node_buf, void* scratch,
                    zha_tree** out) {
  if (!out) return fail(ZHA_ERR_INVALID, "out is NULL");
  *out = nullptr;
  Layout L;
  int rc = make_layout(cfg, &L);
  if (rc) return rc;
  if (!K || !V || !refs || !node_buf || !scratch) return fail(ZHA_ERR_INVALID, "a buffer pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V) | reinterpret_cast<uintptr_t>(refs)) & 15)
    return fail(ZHA_ERR_INVALID, "K, V and refs must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(node_buf) | reinterpret_cast<uintptr_t>(scratch)) & 255)
    return fail(ZHA_ERR_INVALID, "node_buf and scratch must be 256-byte aligned");
  zha_tree* t = new (std::nothrow) zha_tree;
  if (!t) return fail(ZHA_ERR_INVALID, "out of host memory");
  t->cfg = *cfg;
  t->L = L;
  t->scratch = static_cast<char*>(scratch);
  t->n = 0;
  t->spin_limit = kDefaultSpinLimit;
  t->flow_dirty = true;
  t->n_step_p = 0;
  if (const char* v = std::getenv("ZHA_SPIN_LIMIT")) {  // test hook: 0 makes every wait give up at once
    const long long x = std::atoll(v);
    if (x >= 0 && (x > 0 || v[0] == '0')) t->spin_limit = x;
  }
  cudaGetDevice(&t->device);
  TreeDev& d = t->dev;
  std::memset(&d, 0, sizeof(d));
  d.d = cfg->d;
  d.hq = cfg->n_q_heads;
  d.hkv = cfg->n_kv_heads;
  d.group = cfg->n_q_heads / cfg->n_kv_heads;
  d.block = cfg->block;
  d.levels = cfg->levels;
  d.refs = cfg->n_refs;
  d.chunk_level = L.S;
  d.capacity = cfg->capacity;
  for (int l = 0; l <= kMaxLevels; ++l) {
    d.cap_nodes[l] = L.cap_nodes[l];
    d.pow_b[l] = L.pow_b[l];
    d.rec_off[l] = L.rec_off[l];
    d.f_off[l] = L.f_off[l];
    d.up_off[l] = L.up_off[l];
    d.rec4_off[l] = L.rec4_off[l];
  }
  d.rec_bytes = L.rec_bytes;
  d.planes = cfg->planes;
  d.rec4_bytes = L.rec4_bytes;
  d.up_bytes = L.up_bytes;
  d.nodes = static_cast<char*>(node_buf);
  d.K = K;
  d.V = V;
  d.refsp = refs;
  d.status = reinterpret_cast<int*>(t->scratch + L.status_off);
  d.inv_sqrt_d = 1.0f / std::sqrt(float(cfg->d));
  *out = t;
  return ZHA_OK;
}

void zha_tree_destroy(zha_tree* tree) { delete tree; }

int64_t zha_tree_size(const zha_tree* tree) { return tree ? tree->n : -1; }

int zha_tree_build(zha_tree* t, int64_t n, void* stream) {
  if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
  if (n < 0) return fail(ZHA_ERR_INVALID, "n must be >= 0");
  if (n > t->cfg.capacity) return fail(ZHA_ERR_CAPACITY, "n exceeds capacity");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(t->scratch, 0, 256, st);
  if (e != cudaSuccess) return fail_cuda(e, "zha_tree_build: clearing the status word");
  e = launch_tree_update(t->dev, t->cfg.dtype, 0, n, st);
  if (e != cudaSuccess) return fail_cuda(e, "zha_tree_build");
  t->n = n;
  t->flow_dirty = true;
  return ZHA_OK;
}

int zha_tree_append(zha_tree* t, const void* K_new, const void* V_new, int64_t m, void* stream) {
  if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
  if (m < 0) return fail(ZHA_ERR_INVALID, "m must be >= 0");
  if (m == 0) return ZHA_OK;
  if (!K_new || !V_new) return fail(ZHA_ERR_INVALID, "K_new / V_new is NULL");
  if ((reinterpret_cast<uintptr_t>(K_new) | reinterpret_cast<uintptr_t>(V_new)) & 15)
    return fail(ZHA_ERR_INVALID, "K_new and V_new must be 16-byte aligned");
  if (t->n + m > t->cfg.capacity) return fail(ZHA_ERR_CAPACITY, "append exceeds capacity");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (append_fast_ok(t->dev, t->n, m)) {  // no node of levels 2..S completes: copy and new leaves in one kernel
    cudaError_t e = launch_append_fast(t->dev, t->cfg.dtype, K_new, V_new, t->n, m, st);
    if (e != cudaSuccess) return fail_cuda(e, "zha_tree_append: fast path");
    t->n += m;
    return ZHA_OK;
  }
  cudaError_t e = launch_append_copy(t->dev, t->cfg.dtype, K_new, V_new, t->n, m, st);
  if (e != cudaSuccess) return fail_cuda(e, "zha_tree_append: copy");
  e = launch_tree_update(t->dev, t->cfg.dtype, t->n, t->n + m, st);
  if (e != cudaSuccess) return fail_cuda(e, "zha_tree_append: update");
  t->n += m;
  return ZHA_OK;
}

static int fill_decode_args(const zha_tree* t, const void* Q, float* O, int32_t* kept, int32_t* kept_cnt,
                            int64_t* stats, int32_t* scored, int64_t scored_cap, DecodeArgs* a) {
  std::memset(a, 0, sizeof(*a));
  a->t = t->dev;
  a->Q = Q;
  a->O = O;
  a->n_tokens = t->n;
  const int L = t->cfg.levels, b = t->cfg.block;
  for (int l = 0; l <= L; ++l) a->nl[l] = t->n / t->L.pow_b[l];
  int64_t roots = a->nl[L];
  int steps = roots > 0 ? L : 0;
  for (int l = L - 1; l >= 1; --l) {
    const int64_t cnt = a->nl[l] - int64_t(b) * a->nl[l + 1];
    roots += cnt;
    if (cnt > 0 && steps < l) steps = l;
  }
  a->n_roots = int(roots);
  a->n_steps = steps;
  a->ws = t->scratch + t->L.ws_off;
  a->ws_per_bh = t->L.ws_per_bh;
  a->flow = reinterpret_cast<unsigned char*>(t->scratch + t->L.flow_off);
  a->attn_part = reinterpret_cast<float*>(t->scratch + t->L.part_off);
  a->spin_limit = t->spin_limit;
  a->cap_sel = t->L.cap_sel;
  a->cap_list = t->L.cap_list;
  a->kept = kept;
  a->kept_cnt = kept_cnt;
  a->stats = stats;
  a->scored = scored;
  a->scored_cap = scored ? scored_cap : 0;
  a->kept_stride = t->L.cap_nodes[1];
  for (int s = 0; s < kMaxLevels; ++s) {
    const float p = t->n_step_p > 0 ? t->step_p[s < t->n_step_p ? s : t->n_step_p - 1] : t->cfg.p;
    if (p >= 1.f) {
      a->p_all[s] = 1;
    } else {
      int ex = 0;
      const float fr = std::frexp(p, &ex);           // p = fr * 2^ex, fr in [0.5, 1)
      a->p_mant[s] = uint32_t(std::ldexp(fr, 24));   // exact: fr has 24 significant bits
      a->p_shift[s] = 24 - ex;
    }
  }
  return ZHA_OK;
}

int zha_decode(const zha_tree* t, const void* Q, float* O, int32_t B, int32_t* kept, int32_t* kept_cnt,
               int64_t* stats, int32_t* scored, int64_t scored_cap, void* stream) {
  if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
  if (!Q || !O) return fail(ZHA_ERR_INVALID, "Q / O is NULL");
  if ((kept == nullptr) != (kept_cnt == nullptr)) return fail(ZHA_ERR_INVALID, "kept and kept_cnt go together");
  if (B < 1) return fail(ZHA_ERR_INVALID, "B must be >= 1");
  if (B > t->cfg.max_batch) return fail(ZHA_ERR_CAPACITY, "B exceeds max_batch");
  if (t->n < 1) return fail(ZHA_ERR_INVALID, "decode needs at least one cached token");
  if (scored && scored_cap < 1) return fail(ZHA_ERR_INVALID, "scored needs scored_cap >= 1");
  if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(O)) & 15)
    return fail(ZHA_ERR_INVALID, "Q and O must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  zha_tree* tm = const_cast<zha_tree*>(t);
  if (tm->flow_dirty) {  // first decode of this tree, or the first after an error status
    cudaError_t e = cudaMemsetAsync(t->scratch + t->L.flow_off, 0, t->L.flow_bytes, st);
    if (e != cudaSuccess) return fail_cuda(e, "zha_decode: clearing the routing state");
    tm->flow_dirty = false;
  }
  DecodeArgs a;
  fill_decode_args(t, Q, O, kept, kept_cnt, stats, scored, scored_cap, &a);
  a.nheads = B * t->cfg.n_q_heads;
  a.max_heads = t->cfg.max_batch * t->cfg.n_q_heads;
  cudaError_t e = launch_decode(a, t->cfg.dtype, st);
  if (e != cudaSuccess) {
    tm->flow_dirty = true;
    return fail_cuda(e, "zha_decode");
  }
  return ZHA_OK;
}

int zha_route_multi(zha_tree* t, const void* Q, float* O, int32_t m, int32_t* kept, int32_t* kept_cnt,
                    void* stream) {
  if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
  if (!Q || !O) return fail(ZHA_ERR_INVALID, "Q / O is NULL");
  if ((kept == nullptr) != (kept_cnt == nullptr)) return fail(ZHA_ERR_INVALID, "kept and kept_cnt go together");
  if (m < 1) return fail(ZHA_ERR_INVALID, "m must be >= 1");
  if (t->n < 1) return fail(ZHA_ERR_INVALID, "routing needs at least one cached token");
  if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(O)) & 15)
    return fail(ZHA_ERR_INVALID, "Q and O must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int hq = t->cfg.n_q_heads, d = t->cfg.d, es = elem_size(t->cfg.dtype);
  const int64_t cap1 = t->L.cap_nodes[1];
  for (int64_t q0 = 0; q0 < m; q0 += t->cfg.max_batch) {
    const int B = int(min64(t->cfg.max_batch, m - q0));
    if (t->flow_dirty) {
      cudaError_t e = cudaMemsetAsync(t->scratch + t->L.flow_off, 0, t->L.flow_bytes, st);
      if (e != cudaSuccess) return fail_cuda(e, "zha_route_multi: clearing the routing state");
      t->flow_dirty = false;
    }
    DecodeArgs a;
    fill_decode_args(t, static_cast<const char*>(Q) + size_t(q0) * hq * d * es, O + size_t(q0) * hq * d,
                     kept ? kept + size_t(q0) * hq * cap1 : nullptr, kept_cnt ? kept_cnt + size_t(q0) * hq : nullptr,
                     nullptr, nullptr, 0, &a);
    a.nheads = B * hq;
    a.max_heads = t->cfg.max_batch * hq;
    a.root_gemm = t->cfg.dtype == ZHA_BF16 ? 1 : 0;
    cudaError_t e = launch_decode(a, t->cfg.dtype, st);
    if (e != cudaSuccess) {
      t->flow_dirty = true;
      return fail_cuda(e, "zha_route_multi");
    }
  }
  return ZHA_OK;
}

int zha_decode_step_host(zha_tree* t, const void* k_host, const void* v_host, const void* q_host, float* o_host,
                         int32_t B, void* stream) {
  if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
  if (!q_host || !o_host) return fail(ZHA_ERR_INVALID, "q_host / o_host is NULL");
  if ((k_host == nullptr) != (v_host == nullptr)) return fail(ZHA_ERR_INVALID, "k_host and v_host go together");
  if (B < 1 || B > t->cfg.max_batch) return fail(ZHA_ERR_CAPACITY, "B out of range");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int es = elem_size(t->cfg.dtype);
  char* sk = t->scratch + t->L.stage_k;
  char* sv = t->scratch + t->L.stage_v;
  char* sq = t->scratch + t->L.stage_q;
  float* so = reinterpret_cast<float*>(t->scratch + t->L.stage_o);
  const size_t kv_bytes = size_t(t->cfg.n_kv_heads) * t->cfg.d * es;
  const size_t q_bytes = size_t(B) * t->cfg.n_q_heads * t->cfg.d * es;
  const size_t o_bytes = size_t(B) * t->cfg.n_q_heads * t->cfg.d * 4;
  cudaError_t e;
  if (k_host) {
    if ((e = cudaMemcpyAsync(sk, k_host, kv_bytes, cudaMemcpyHostToDevice, st)) != cudaSuccess)
      return fail_cuda(e, "zha_decode_step_host: K copy");
    if ((e = cudaMemcpyAsync(sv, v_host, kv_bytes, cudaMemcpyHostToDevice, st)) != cudaSuccess)
      return fail_cuda(e, "zha_decode_step_host: V copy");
  }
  if ((e = cudaMemcpyAsync(sq, q_host, q_bytes, cudaMemcpyHostToDevice, st)) != cudaSuccess)
    return fail_cuda(e, "zha_decode_step_host: Q copy");
  int rc;
  if (k_host && (rc = zha_tree_append(t, sk, sv, 1, stream)) != ZHA_OK) return rc;
  if ((rc = zha_decode(t, sq, so, B, nullptr, nullptr, nullptr, nullptr, 0, stream)) != ZHA_OK) return rc;
  if ((e = cudaMemcpyAsync(o_host, so, o_bytes, cudaMemcpyDeviceToHost, st)) != cudaSuccess)
    return fail_cuda(e, "zha_decode_step_host: O copy");
  return ZHA_OK;
}

// Split partials of any dense decode with B' <= B sequences over n' <= n tokens.  dense_plan gives
// splits' <= min(ceil(X / B'), ceil(n' / 64)) with X = ceil(dense_target / Hkv) (its split count is not
// monotone in n, so the bound is taken over the plan's caps, not over one plan): B' * ceil(X / B') <=
// X + B' - 1 <= X + B - 1, and B' * ceil(n' / 64) <= B * ceil(n / 64).
static uint64_t dense_part_floats_bound(const zha_config* cfg, int32_t B, int64_t n) {
  const uint64_t X = (uint64_t(dense_target_splits()) + cfg->n_kv_heads - 1) / cfg->n_kv_heads;
  const uint64_t by_target = X + uint64_t(B) - 1;
  const uint64_t by_len = uint64_t(B) * uint64_t((n + 63) / 64);
  const uint64_t seq_splits = by_target < by_len ? by_target : by_len;  // bound on B' * splits'
  return uint64_t(cfg->n_q_heads) * seq_splits * uint64_t(cfg->d + 2);
}

size_t zha_dense_scratch_bytes(const zha_config* cfg, int32_t B, int64_t n) {
  if (validate(cfg) || B < 1 || n < 1 || B > cfg->max_batch) return 0;
  return size_t(align256(dense_part_floats_bound(cfg, B, n) * 4));
}

int zha_dense_decode(const zha_config* cfg, const void* K, const void* V, int64_t ld, int64_t n, const void* Q,
                     float* O, int32_t B, void* scratch, void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  if (!K || !V || !Q || !O || !scratch) return fail(ZHA_ERR_INVALID, "a pointer is NULL");
  if (n < 1 || ld < n) return fail(ZHA_ERR_INVALID, "need 1 <= n <= ld");
  if (B < 1) return fail(ZHA_ERR_INVALID, "B must be >= 1");
  if (B > cfg->max_batch) return fail(ZHA_ERR_CAPACITY, "B exceeds max_batch");
  if ((reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V) | reinterpret_cast<uintptr_t>(Q) |
       reinterpret_cast<uintptr_t>(O)) & 15)
    return fail(ZHA_ERR_INVALID, "K, V, Q and O must be 16-byte aligned");
  DenseArgs a;
  std::memset(&a, 0, sizeof(a));
  dense_plan(B, cfg->n_kv_heads, n, &a.splits, &a.per);
  a.K = K;
  a.V = V;
  a.Q = Q;
  a.O = O;
  a.part = static_cast<float*>(scratch);
  a.ld = ld;
  a.n = n;
  a.hq = cfg->n_q_heads;
  a.hkv = cfg->n_kv_heads;
  a.group = cfg->n_q_heads / cfg->n_kv_heads;
  a.inv_sqrt_d = 1.0f / std::sqrt(float(cfg->d));
  cudaError_t e = launch_dense(a, cfg->dtype, cfg->d, B, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "zha_dense_decode");
  return ZHA_OK;
}

// Dense decode for callers that cannot allocate device memory: the split
// partials go to the library's fixed static array (see zha.h).
int zha_dense_decode_noalloc(const zha_config* cfg, const void* K, const void* V, int64_t ld, int64_t n,
                             const void* Q, float* O, int32_t B, void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  if (!K || !V || !Q || !O) return fail(ZHA_ERR_INVALID, "a pointer is NULL");
  if (n < 1 || ld < n) return fail(ZHA_ERR_INVALID, "need 1 <= n <= ld");
  if (B < 1) return fail(ZHA_ERR_INVALID, "B must be >= 1");
  if (B > cfg->max_batch) return fail(ZHA_ERR_CAPACITY, "B exceeds max_batch");
  if ((reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V) | reinterpret_cast<uintptr_t>(Q) |
       reinterpret_cast<uintptr_t>(O)) & 15)
    return fail(ZHA_ERR_INVALID, "K, V, Q and O must be 16-byte aligned");
  DenseArgs a;
  std::memset(&a, 0, sizeof(a));
  dense_plan(B, cfg->n_kv_heads, n, &a.splits, &a.per);
  const uint64_t floats = uint64_t(B) * cfg->n_q_heads * a.splits * (cfg->d + 2);
  if (floats > dense_static_floats())
    return fail(ZHA_ERR_CAPACITY, "B * n_q_heads * splits * (d + 2) exceeds the fixed scratch of 2^20 floats");
  float* part = nullptr;
  cudaError_t e = dense_static_scratch(&part);
  if (e != cudaSuccess) return fail_cuda(e, "zha_dense_decode_noalloc: looking up the fixed scratch");
  a.K = K;
  a.V = V;
  a.Q = Q;
  a.O = O;
  a.part = part;
  a.ld = ld;
  a.n = n;
  a.hq = cfg->n_q_heads;
  a.hkv = cfg->n_kv_heads;
  a.group = cfg->n_q_heads / cfg->n_kv_heads;
  a.inv_sqrt_d = 1.0f / std::sqrt(float(cfg->d));
  e = launch_dense(a, cfg->dtype, cfg->d, B, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "zha_dense_decode_noalloc");
  return ZHA_OK;
}

int zha_tree_set_step_p(zha_tree* t, const float* p, int32_t n) {
  if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
  if (n < 0 || n > kMaxLevels) return fail(ZHA_ERR_INVALID, "n must be in 0..20");
  if (n > 0 && !p) return fail(ZHA_ERR_INVALID, "p is NULL");
  for (int i = 0; i < n; ++i)
    if (!(p[i] > 0.f) || !(p[i] <= 1.f)) return fail(ZHA_ERR_INVALID, "every threshold must be in (0, 1]");
  for (int i = 0; i < n; ++i) t->step_p[i] = p[i];
  t->n_step_p = n;
  return ZHA_OK;
}

int zha_tree_status(zha_tree* t, void* stream) {
  if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail_cuda(e, "zha_tree_status: synchronize");
  int status = 0;
  e = cudaMemcpy(&status, t->dev.status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail_cuda(e, "zha_tree_status: read");
  if (status != 0) {
    const int zero = 0;
    cudaMemcpy(t->dev.status, &zero, sizeof(int), cudaMemcpyHostToDevice);
    t->flow_dirty = true;  // a kernel that gave up may have left the routing state mid-way
    switch (status) {
      case ZHA_ERR_CAPACITY:
        return fail(status, "a kernel raised ZHA_ERR_CAPACITY (a capacity bound would have been exceeded)");
      case ZHA_ERR_TIMEOUT:
        return fail(status, "a kernel raised ZHA_ERR_TIMEOUT (a bounded wait on a copy ran out)");
      default:
        return fail(status, "a kernel raised an unknown error status");
    }
  }
  return ZHA_OK;
}

}  // extern "C"
