// C ABI of the dynamic hashed embedding engine (see include/dhs.h).
//
// Host side: table lifecycle, growth of the IDMap (rehash of keys and
// offsets only; rows never move) and of the EmbeddingBlocks (append), the
// per-call workspace, and the launch sequence of each call.  Every step of
// every call runs in the kernels of dhs_fwd.cuh / dhs_bwd.cuh; the host only
// sizes, allocates and launches.
#include <cuda_runtime.h>

#include <algorithm>
#include <chrono>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <new>
#include <vector>

#include "../../include/dhs.h"
#include "dhs_bwd.cuh"
#include "dhs_device.cuh"
#include "dhs_fwd.cuh"
#include "dhs_launch.h"
#include "dhs_shard.cuh"

using namespace dhs;

namespace dhs {

int blocks_per_sm(const void* kernel, int threads, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int, size_t>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_tuple(kernel, dev, threads, smem);
  std::lock_guard<std::mutex> lock(mu);
  const auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  // opt in to the dynamic size asked for: static + dynamic shared memory above
  // 48 KB needs it even when the dynamic part alone is below
  if (smem > 0) cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess || per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  }
  cache.emplace(key, per_sm);
  return per_sm;
}

}  // namespace dhs

namespace {

constexpr long long kDefaultBlockRows = 1ll << 20;
constexpr long long kDefaultMaxRows = 1ll << 31;
constexpr long long kMaxRowsLimit = (1ll << 32) - 2;
constexpr unsigned long long kInitialSlots = 1ull << 16;
constexpr double kMaxLoad = 0.5;
// Sort chunk of the segment-reduce kernel: big enough that a group's fixed
// work per chunk stays small, small enough that every SM gets many chunks.
int seg_chunk(long long n) {
#ifdef DHS_SEG_CHUNK_FIXED  // tuning override (a power of two >= 32)
  if (n > 100000) return DHS_SEG_CHUNK_FIXED;
#endif
  return n > 100000 ? 64 : 32;
}
constexpr int kSnapRing = 4;
enum { PH_FWD_POOL = 0, PH_FWD_ASSIGN = 1, PH_BWD_PROBE = 2, PH_BWD_SORT = 3, PH_BWD_SEG = 4,
       PH_LOOKUP_INSERT = 5, PH_GROW = 6, PH_FWD_PROBE = 7, PH_BWD_COMBINE = 8 };

struct Snap {
  cudaEvent_t ev = nullptr;
  unsigned long long* pinned = nullptr;  // row_count, keys_used, sum_unique written here (mapped)
  unsigned long long* pinned_dev = nullptr;  // the same memory as the device addresses it
  long long cum_n = 0;                   // inserted-key upper bound counter at record time
  long long bwd_n = 0;                   // ids of all backward calls enqueued before it
  bool valid = false;
};

struct PhaseRec {
  int phase;
  cudaEvent_t a, b;
};

struct Buf {
  void* p = nullptr;
  size_t bytes = 0;
};

int pick_group(int dim) {
  int need = (dim + 3) / 4;
  int g = 1;
  while (g < need && g < 32) g <<= 1;
  return g;
}

// float4 columns per lane: 1, 2 or 4 (the kernels are instantiated for these)
int pick_nv(int dim, int g) {
  const int need = (dim / 4 + g - 1) / g;
  int v = 1;
  while (v < need) v <<= 1;
  return v;
}

// Segment-kernel lanes: 8 float columns per lane (two float4), so that a
// warp holds two or more groups and the per-pair control work is shared;
// rows wider than 256 floats use 16 columns per lane.
int seg_group(int dim) {
  if (dim > 256) return 32;
  const int need = (dim + 7) / 8;
  int g = 1;
  while (g < need) g <<= 1;
  return g;
}

int seg_nv(int dim) { return dim > 256 ? 4 : 2; }

int log2_exact(long long x) {
  int l = 0;
  while ((1ll << l) < x) ++l;
  return l;
}

}  // namespace

struct dhs_table {
  int device = 0;
  int sm_count = 148;
  int dim = 0, opt = 0, stride = 0;
  int wfl = 0;          // floats per row holding the weights (dim, or dim / 2 for bf16 weights)
  bool wbf16 = false;   // weights stored as bf16
  float eps = 1e-8f, b1 = 0.9f, b2 = 0.999f;
  long long adam_t = 0;
  long long block_rows = kDefaultBlockRows;
  int log2_br = 20;
  long long max_rows = kDefaultMaxRows;
  long long max_blocks = 0;
  dhs_allocator alloc{};
  bool custom_alloc = false;
  cudaMemPool_t pool = nullptr;  // table-owned stream-ordered pool (keeps freed memory)
  cudaStream_t last_stream = nullptr;

  Slot* slots = nullptr;
  unsigned long long nslots = 0;
  long long n_rehash = 0;
  long long n_insert_calls = 0;
  long long n_pool_calls = 0;  // fused pool launches (their chunk counters alternate)
  long long n_launches = 0;  // kernels launched by this table's calls
  long long n_host_waits = 0, host_wait_ns = 0;  // host blocked on the device
  long long n_allocs = 0, alloc_ns = 0;          // device allocations

  std::vector<float*> blocks_h;
  float** blocks_d = nullptr;
  DevState* st = nullptr;

  // upper bound on the device row count after all enqueued work
  long long rows_ub = 0;
  // with hooks: upper bound on the IDMap slots in use (keys with or without a
  // row, and tombstones until the next rehash)
  long long keys_ub = 0;

  // admission / eviction (ht_set_hooks)
  bool has_hooks_set = false;
  unsigned admit = 1;
  bool track = false;
  long long step = 0;          // insert calls so far
  unsigned* cnt = nullptr;     // [nslots]
  unsigned* stamp = nullptr;   // [nslots]
  unsigned* free_bm = nullptr; // bit per row
  long long free_words = 0;
  unsigned* free_list = nullptr;
  long long free_list_cap = 0;
  Buf b_fcnt, b_freed;
  long long cum_n = 0;  // sum of key counts of all insert calls
  long long bwd_n = 0;  // sum of key counts of all backward calls
  // from the newest finished snapshot: ids of the backward calls before it
  // and the distinct rows they updated (their ratio is the mean segment length)
  long long seen_bwd_n = 0, seen_unique = 0;
  Snap snaps[kSnapRing];
  int snap_next = 0;

  // workspace, sized for ws_n positions
  long long ws_n = -1;
  long long ws_chunks = 0;  // chunk capacity of the segment and combine buffers
  Buf b_nbm, b_fbm, b_gcnt, b_gpref, b_slotpos, b_ka, b_va, b_kb, b_vb, b_hist, b_totals, b_ph,
      b_pt, b_owners, b_cplan, b_slots, b_refs, b_bagpos, b_mult, b_runs, b_shard, b_reckey;
  long long ws_run_cap = 0;  // entries of the long-segment arrival table
  // positions of the last insert call when it was a split forward, whose
  // keys (b_reckey) and rows (b_refs) are recorded per position; -1: none
  long long rec_n = -1;
  int hist_sel = 0;          // which half of b_hist the next backward uses (the probe clears the other)

  int timing = 0;  // 0 off, 1 every phase, 2 the IDMap growth phase only
  std::vector<PhaseRec> recs;
  std::vector<cudaEvent_t> ev_pool;
};

namespace {

long long now_ns() {
  return std::chrono::duration_cast<std::chrono::nanoseconds>(
             std::chrono::steady_clock::now().time_since_epoch())
      .count();
}

void* dalloc(dhs_table* t, size_t bytes, cudaStream_t s) {
  if (bytes == 0) bytes = 16;
  const long long t0 = now_ns();
  void* p = nullptr;
  if (t->custom_alloc) {
    p = t->alloc.alloc(bytes, (dhs_stream)s, t->alloc.ctx);
  } else if (cudaMallocFromPoolAsync(&p, bytes, t->pool, s) != cudaSuccess) {
    cudaGetLastError();
    p = nullptr;
  }
  t->n_allocs++;
  t->alloc_ns += now_ns() - t0;
  return p;
}

cudaError_t host_wait(dhs_table* t, cudaEvent_t ev) {
  const long long t0 = now_ns();
  const cudaError_t e = cudaEventSynchronize(ev);
  t->n_host_waits++;
  t->host_wait_ns += now_ns() - t0;
  return e;
}

void dfree(dhs_table* t, void* p, size_t bytes, cudaStream_t s) {
  if (!p) return;
  if (t->custom_alloc)
    t->alloc.free(p, bytes ? bytes : 16, (dhs_stream)s, t->alloc.ctx);
  else
    cudaFreeAsync(p, s);
}

dhs_status bget(dhs_table* t, Buf& b, size_t bytes, cudaStream_t s) {
  if (b.bytes >= bytes && b.p) return DHS_OK;
  dfree(t, b.p, b.bytes, s);
  b.p = dalloc(t, bytes, s);
  b.bytes = b.p ? bytes : 0;
  return b.p ? DHS_OK : DHS_ERR_OOM;
}

void bfree(dhs_table* t, Buf& b, cudaStream_t s) {
  dfree(t, b.p, b.bytes, s);
  b.p = nullptr;
  b.bytes = 0;
}

size_t block_bytes(const dhs_table* t) { return (size_t)t->block_rows * t->stride * sizeof(float); }

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    int cur = -1;
    if (cudaGetDevice(&cur) == cudaSuccess && cur != dev) {
      prev = cur;
      cudaSetDevice(dev);
    }
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

dhs_status last_launch() {
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return DHS_OK;
  return e == cudaErrorMemoryAllocation ? DHS_ERR_OOM : DHS_ERR_CUDA;
}

#define DHS_TRY(x)                  \
  do {                              \
    dhs_status _s = (x);            \
    if (_s != DHS_OK) return _s;    \
  } while (0)

#define DHS_CUDA(x)                                         \
  do {                                                      \
    if ((x) != cudaSuccess) {                               \
      cudaGetLastError();                                   \
      return DHS_ERR_CUDA;                                  \
    }                                                       \
  } while (0)

IdMap idmap(const dhs_table* t) { return IdMap{t->slots, t->nslots / 2 - 1}; }

RowSpace rowspace(const dhs_table* t) {
  return RowSpace{t->blocks_d, (unsigned long long)t->block_rows - 1, t->log2_br, t->stride, t->wfl};
}

bool has_hooks(const dhs_table* t) { return t->admit > 1 || t->track; }

Hooks hooks(const dhs_table* t) {
  return Hooks{t->admit > 1 ? t->cnt : nullptr, t->track ? t->stamp : nullptr, t->admit, (unsigned)t->step,
               t->free_list, t->free_bm};
}

// ---- phase timing ----
cudaEvent_t ev_get(dhs_table* t) {
  if (!t->ev_pool.empty()) {
    cudaEvent_t e = t->ev_pool.back();
    t->ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct PhaseScope {
  dhs_table* t;
  int phase;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  PhaseScope(dhs_table* t_, int ph, cudaStream_t s_) : t(t_), phase(ph), s(s_) {
    if (t->timing == 1 || (t->timing == 2 && ph == PH_GROW)) {
      a = ev_get(t);
      cudaEventRecord(a, s);
    }
  }
  ~PhaseScope() {
    if (a) {
      cudaEvent_t b = ev_get(t);
      cudaEventRecord(b, s);
      t->recs.push_back(PhaseRec{phase, a, b});
    }
  }
};

// ---- grid sizing ----
template <typename K>
int resident_blocks(K kernel, int threads, size_t smem, int sm_count) {
  return blocks_per_sm((const void*)kernel, threads, smem) * sm_count;
}

long long grid_for(long long units_per_block_needed, int resident) {
  if (units_per_block_needed < 1) return 1;
  return std::min<long long>(units_per_block_needed, resident);
}

// ---- row-count bookkeeping ----
// Use the newest finished snapshot of the device row count to tighten the
// host's upper bound; with `wait`, wait for the newest recorded snapshot.
void refresh_ub(dhs_table* t, bool wait) {
  for (int i = 0; i < kSnapRing; ++i) {
    const int k = ((t->snap_next - 1 - i) % kSnapRing + kSnapRing) % kSnapRing;
    Snap& sn = t->snaps[k];
    if (!sn.valid) continue;
    cudaError_t q = wait && i == 0 ? host_wait(t, sn.ev) : cudaEventQuery(sn.ev);
    if (q == cudaSuccess) {
      const long long ub = (long long)sn.pinned[0] + (t->cum_n - sn.cum_n);
      if (ub < t->rows_ub) t->rows_ub = ub;
      const long long kb = (long long)sn.pinned[1] + (t->cum_n - sn.cum_n);
      if (kb < t->keys_ub) t->keys_ub = kb;
      t->seen_bwd_n = sn.bwd_n;
      t->seen_unique = (long long)sn.pinned[2];
      return;
    }
    cudaGetLastError();
  }
}

// The device's row count and key count written straight into mapped pinned
// host memory (no copy-engine transfer on the stream: a one-warp kernel).
__global__ void snapshot_kernel(const DevState* st, volatile unsigned long long* host) {
  pdl_enter();
  if (threadIdx.x == 0) {
    host[0] = st->row_count;
    host[1] = st->keys_used;
    host[2] = st->sum_unique;
    __threadfence_system();
  }
}

void record_snapshot(dhs_table* t, cudaStream_t s) {
  Snap& sn = t->snaps[t->snap_next];
  if (sn.valid) host_wait(t, sn.ev);  // ring slot reuse: at most kSnapRing in flight
  launch_k(snapshot_kernel, 1, 32, 0, s, t->st, sn.pinned_dev);
  t->n_launches++;
  cudaEventRecord(sn.ev, s);
  sn.cum_n = t->cum_n;
  sn.bwd_n = t->bwd_n;
  sn.valid = true;
  t->snap_next = (t->snap_next + 1) % kSnapRing;
}

__global__ void set_block_kernel(float** blocks_d, long long idx, float* ptr, DevState* st,
                                 unsigned long long n_blocks) {
  blocks_d[idx] = ptr;
  st->n_blocks = n_blocks;
}

dhs_status grow_map(dhs_table* t, unsigned long long want_slots, cudaStream_t s) {
  PhaseScope ph(t, PH_GROW, s);
  unsigned long long ns = std::max<unsigned long long>(t->nslots * 2, kInitialSlots);
  while (ns < want_slots) ns <<= 1;
  const int thr = 256;
  Slot* fresh = (Slot*)dalloc(t, ns * sizeof(Slot), s);
  if (!fresh) return DHS_ERR_OOM;
  const long long g = std::min<long long>((long long)((ns + thr - 1) / thr), (long long)t->sm_count * 16);
  fill_empty_kernel<<<(unsigned)g, thr, 0, s>>>(fresh, ns);
  t->n_launches++;
  // per-slot counts and stamps of the new map (hooks), zero until the rehash
  // moves the keys' values over
  unsigned* ncnt = nullptr;
  unsigned* nstamp = nullptr;
  if (t->cnt) {
    ncnt = (unsigned*)dalloc(t, ns * 4, s);
    if (!ncnt) return DHS_ERR_OOM;
    DHS_CUDA(cudaMemsetAsync(ncnt, 0, ns * 4, s));
  }
  if (t->stamp) {
    nstamp = (unsigned*)dalloc(t, ns * 4, s);
    if (!nstamp) return DHS_ERR_OOM;
    DHS_CUDA(cudaMemsetAsync(nstamp, 0, ns * 4, s));
  }
  if (t->slots) {
    IdMap to{fresh, ns / 2 - 1};
    if (has_hooks(t)) DHS_CUDA(cudaMemsetAsync(&t->st->keys_used, 0, sizeof(unsigned long long), s));
    const long long g2 = std::min<long long>((long long)((t->nslots + thr - 1) / thr), (long long)t->sm_count * 16);
    rehash_kernel<<<(unsigned)g2, thr, 0, s>>>(t->slots, t->nslots, to, t->cnt, ncnt, t->stamp, nstamp, t->st);
    t->n_launches++;
    dfree(t, t->slots, t->nslots * sizeof(Slot), s);
    t->n_rehash++;
  }
  if (t->cnt) dfree(t, t->cnt, t->nslots * 4, s);
  if (t->stamp) dfree(t, t->stamp, t->nslots * 4, s);
  t->cnt = ncnt;
  t->stamp = nstamp;
  t->slots = fresh;
  t->nslots = ns;
  return last_launch();
}

// Make room for up to `n` new keys: IDMap load <= kMaxLoad and blocks
// covering the row upper bound.  The bound is the newest row-count snapshot
// that has finished plus every key of the insert calls enqueued since.  When
// that bound says the table might have to grow (or cross max_rows), the host
// first waits for the newest snapshot (the previous insert call's row count)
// and grows only if the tightened bound still needs it: growth, which maps
// fresh device memory, happens only for rows that can really arrive.
dhs_status ensure_capacity(dhs_table* t, long long n, cudaStream_t s) {
  refresh_ub(t, false);
  long long need = t->rows_ub + n;
  // slots: with hooks, keys without a row and tombstones take slots too
  long long need_slots = has_hooks(t) ? t->keys_ub + n : need;
  const long long have_rows = (long long)t->blocks_h.size() * t->block_rows;
  if (need > t->max_rows || (double)need_slots > kMaxLoad * (double)t->nslots || need > have_rows) {
    refresh_ub(t, true);
    need = t->rows_ub + n;
    need_slots = has_hooks(t) ? t->keys_ub + n : need;
    if (need > t->max_rows) return DHS_ERR_TABLE_FULL;
  }
  if ((double)need_slots > kMaxLoad * (double)t->nslots)
    DHS_TRY(grow_map(t, (unsigned long long)std::ceil((double)need_slots / kMaxLoad), s));
  long long have = (long long)t->blocks_h.size() * t->block_rows;
  while (need > have) {
    if ((long long)t->blocks_h.size() >= t->max_blocks) return DHS_ERR_TABLE_FULL;
    float* b = (float*)dalloc(t, block_bytes(t), s);
    if (!b) return DHS_ERR_OOM;
    t->blocks_h.push_back(b);
    set_block_kernel<<<1, 1, 0, s>>>(t->blocks_d, (long long)t->blocks_h.size() - 1, b, t->st,
                                     (unsigned long long)t->blocks_h.size());
    t->n_launches++;
    DHS_TRY(last_launch());
    have += t->block_rows;
  }
  return DHS_OK;
}

// Capacities of the long-segment combine for a workspace of `nchunks` chunks.
// Owner chunks are at least two apart (a long segment reaches two chunks past
// its owner), so there are at most nchunks / 2 + 1 of them; the runs overlap
// in at most one chunk, so their pieces add up to at most 1.5 nchunks + 1.
// A run of n pieces gets ceil(n / P) batches, P >= kCombineMinPieces: batch
// ids are at most one per run plus pieces / kCombineMinPieces.  Slots: only
// runs of more than one batch take them (n > P), fewer than 2 n / P each.
constexpr long long combine_batch_cap(long long nchunks) {
  return nchunks / 2 + 2 * nchunks / kCombineMinPieces + 64;
}
constexpr long long combine_slot_cap(long long nchunks) { return 4 * nchunks / kCombineMinPieces + 64; }

// Entries of the arrival table of a backward over nchunks sort chunks: a
// power of two of at least nchunks + 2, so that the long segments (each spans
// three chunks or more, so there are at most nchunks / 2 + 1) fill at most
// about half of it.
long long run_table_cap(long long nchunks) {
  long long c = 64;
  while (c < nchunks + 2) c <<= 1;
  return c;
}
// Pieces of a long segment that the segment kernel's warp adds itself; longer
// segments go to the combine kernels.
constexpr unsigned kSegFinishPieces = DHS_SEG_FINISH_PIECES;

// The plan arrays cut from one buffer of 6 nchunks + batch cap words.
CombinePlan combine_plan(unsigned* words, double* slots, long long nchunks, unsigned* zeroed) {
  CombinePlan pl;
  pl.key = words;
  pl.kend = words + nchunks;
  pl.boff = words + 2 * nchunks;
  pl.sbase = words + 3 * nchunks;
  pl.ticket = words + 4 * nchunks;
  pl.ppb = words + 5 * nchunks;
  pl.batch_owner = words + 6 * nchunks;
  pl.slots = slots;
  pl.batch_cap = (unsigned)combine_batch_cap(nchunks);
  pl.slot_cap = (unsigned)combine_slot_cap(nchunks);
  pl.owner_cap = (unsigned)nchunks;
  pl.batch_ctr = zeroed + kCombineBatchCtrWord;
  pl.slot_ctr = zeroed + kCombineSlotCtrWord;
  return pl;
}

dhs_status ensure_ws(dhs_table* t, long long n, cudaStream_t s) {
  if (n <= t->ws_n) return DHS_OK;
  t->rec_n = -1;  // the record does not survive a reallocation
  long long cap = std::max<long long>(n, t->ws_n > 0 ? t->ws_n + t->ws_n / 2 : 0);
  cap = std::max<long long>(cap, 4096);
  const long long ngroups = (cap + kGroupPositions - 1) / kGroupPositions + 1;
  const long long nwords = ngroups * kGroupWords;
  const long long ntiles = (cap + kRadixTile - 1) / kRadixTile;
  const long long nchunks = (cap + seg_chunk(cap) - 1) / seg_chunk(cap) + (cap + 31) / 32;
  const long long pstride = (long long)seg_nv(t->dim) * seg_group(t->dim) * 4;
  DHS_TRY(bget(t, t->b_nbm, nwords * 4, s));
  DHS_TRY(bget(t, t->b_fbm, nwords * 4, s));
  DHS_TRY(bget(t, t->b_gcnt, ngroups * 4, s));
  DHS_TRY(bget(t, t->b_gpref, ngroups * 4, s));
  DHS_TRY(bget(t, t->b_slotpos, cap * 4, s));
  DHS_TRY(bget(t, t->b_refs, cap * 8, s));
  DHS_TRY(bget(t, t->b_reckey, cap * 8, s));
  DHS_TRY(bget(t, t->b_ka, cap * 4, s));
  DHS_TRY(bget(t, t->b_va, cap * 4, s));
  DHS_TRY(bget(t, t->b_kb, cap * 4, s));
  DHS_TRY(bget(t, t->b_vb, cap * 4, s));
  // digit histograms of every pass + one tile counter per pass; look-back state
  // two areas of counters (digit histograms, tile and chunk counters): a
  // backward uses one while its probe clears the other for the next backward
  if (!t->b_hist.p) {
    DHS_TRY(bget(t, t->b_hist, (size_t)2 * kSortZeroWords * 4, s));
    DHS_CUDA(cudaMemsetAsync(t->b_hist.p, 0, t->b_hist.bytes, s));
  }
  DHS_TRY(bget(t, t->b_totals, (size_t)kRadixMaxPasses * ntiles * kRadixBins * 8, s));
  DHS_TRY(bget(t, t->b_ph, (size_t)nchunks * pstride * 8, s));
  DHS_TRY(bget(t, t->b_pt, (size_t)nchunks * pstride * 8, s));
  DHS_TRY(bget(t, t->b_owners, nchunks * 4, s));
  DHS_TRY(bget(t, t->b_cplan, (size_t)(6 * nchunks + combine_batch_cap(nchunks)) * 4, s));
  DHS_TRY(bget(t, t->b_slots, (size_t)combine_slot_cap(nchunks) * pstride * 8, s));
  // arrival table: key, ctr, c0, c1 arrays of run_table_cap entries each
  const long long rcap = run_table_cap(nchunks);
  DHS_TRY(bget(t, t->b_runs, (size_t)4 * rcap * 4, s));
  t->ws_run_cap = rcap;
  DHS_CUDA(cudaMemsetAsync(t->b_nbm.p, 0, t->b_nbm.bytes, s));
  t->ws_n = cap;
  t->ws_chunks = nchunks;
  return DHS_OK;
}

// The per-position bag and factor arrays of an extended-pooling backward
// (allocated on first use, sized like the rest of the workspace).
dhs_status ensure_ws_ext(dhs_table* t, cudaStream_t s) {
  DHS_TRY(bget(t, t->b_bagpos, (size_t)t->ws_n * 4, s));
  return bget(t, t->b_mult, (size_t)t->ws_n * 8, s);
}

dhs_status check_table(const dhs_table* t) { return t ? DHS_OK : DHS_ERR_INVALID_ARG; }

// Floats per row as ht_get_rows / ht_export return it: dim weights (widened
// from bf16 where stored so) followed by the fp32 state.
int export_stride(const dhs_table* t) { return t->dim + (t->stride - t->wfl); }

// Plan and combine launches for the long segments of one backward.
dhs_status launch_combine(dhs_table* t, const unsigned* skey, long long n, const OptArgs& oa,
                          const double* part_head, const double* part_tail, int chunk, int pstride,
                          const unsigned* owners, unsigned* zeroed, const CombinePlan& pl,
                          cudaStream_t s) {
  const unsigned* owner_ctr = zeroed + kSegOwnerCtrWord;
  launch_k(bwd_combine_plan_kernel, (unsigned)t->sm_count * 2, 256, 0, s,
      skey, n, chunk, owners, owner_ctr, pl, t->dim, rowspace(t), oa, part_head, part_tail, pstride, t->st);
  t->n_launches++;
  DHS_TRY(last_launch());
  const size_t smem = (size_t)std::max(kCombineThreads, t->dim) * sizeof(double);
  launch_k(bwd_combine_kernel, (unsigned)t->sm_count * 8, kCombineThreads, smem, s,
      skey, t->dim, rowspace(t), oa, part_head, part_tail, chunk, pstride, owners, owner_ctr, pl);
  t->n_launches++;
  return last_launch();
}

// ---- kernel dispatch on the row width ----
dhs_status dispatch_pool(dhs_table* t, const long long* keys, long long n, const long long* bo,
                         long long nb, const float* psw, bool mean, float* out, cudaStream_t s) {
  // a lane's 16-byte unit holds 4 fp32 or 8 bf16 weights
  const int wd = t->wbf16 ? t->dim / 2 : t->dim;
  const int G = pick_group(wd), NV = pick_nv(wd, G);
  const cudaError_t e =
      (t->wbf16 ? launch_probe_pool_bf16 : launch_probe_pool)(G, NV, t->sm_count, idmap(t), rowspace(t), t->dim,
                                                              keys, n, bo, nb, psw, mean, out,
                                                              (unsigned*)t->b_nbm.p, (unsigned*)t->b_slotpos.p,
                                                              (int)(t->n_pool_calls & 1), t->st, s);
  t->n_launches++;
  if (e != cudaSuccess) {
    cudaGetLastError();
    return DHS_ERR_CUDA;
  }
  t->n_pool_calls++;  // the launch cleared the other counter for the next one
  return DHS_OK;
}

// Bags per warp of the backward probe: 64 when bags are short (two positions
// per lane come from different bags), 32 when they are long (more warps).
int bwd_probe_bags(long long n_keys, long long n_bags) { return n_keys < 4 * n_bags ? 64 : 32; }

// Segment kernel for one backward: the warp-per-chunk kernel for rows of at
// least DHS_SEGW_MIN_DIM floats, the lane-group kernel below that.
int segw_cpl(int dim) {
  int c = 1;
  while (32 * c < dim) c *= 2;
  return c;
}

// The segment kernel for a backward: the lane-group kernel for rows of fewer
// than DHS_SEGW_MIN_DIM floats, and for fp32 rows of more than that and at
// most DHS_SEG_NARROW_MAX_DIM floats while the table's segments have been
// short (fewer than DHS_SEG_NARROW_RUN ids per distinct row over its backward
// calls so far): a warp per chunk spends most of its issue slots on
// per-segment work there.  Otherwise the warp-per-chunk kernel.
bool use_narrow_seg(const dhs_table* t) {
  if (t->dim < DHS_SEGW_MIN_DIM) return true;
  return !t->wbf16 && t->dim > DHS_SEGW_MIN_DIM && t->dim <= DHS_SEG_NARROW_MAX_DIM && t->seen_unique > 0 &&
         t->seen_bwd_n < (long long)DHS_SEG_NARROW_RUN * t->seen_unique;
}

// bagpos / mult non-null: extended pooling (sort values are positions).
dhs_status launch_seg(dhs_table* t, const unsigned* sk, const unsigned* sv, long long n, const float* grad,
                      long long nb, const OptArgs& oa, double* part_head, double* part_tail,
                      unsigned* chunk_ctr, unsigned* owners, unsigned* owner_ctr, const unsigned* bagpos,
                      const double* mult, bool mean, const RunTable& rt, cudaStream_t s) {
  const int G = seg_group(t->dim), NV = seg_nv(t->dim);
  const int pstride = NV * G * 4;  // doubles per partial (>= dim)
  const bool ext = mult != nullptr;
  cudaError_t e;
  if (!use_narrow_seg(t)) {
    auto fn = t->opt == DHS_SGD ? (ext ? launch_seg_sgd_ext_w : launch_seg_sgd_w)
              : t->opt == DHS_ADAGRAD ? (ext ? launch_seg_adagrad_ext_w : launch_seg_adagrad_w)
              : t->opt == DHS_ADAM ? (ext ? launch_seg_adam_ext_w : launch_seg_adam_w)
                                   : (ext ? launch_seg_rowwise_ext_w : launch_seg_rowwise_w);
    e = fn(segw_cpl(t->dim), t->wbf16, t->sm_count, sk, sv, n, grad, nb, t->dim, rowspace(t), oa, part_head,
           part_tail, pstride, seg_chunk(n), chunk_ctr, owners, owner_ctr, t->st, bagpos, mult, mean, rt, s);
  } else {
    auto fn = t->opt == DHS_SGD ? (ext ? launch_seg_sgd_ext : launch_seg_sgd)
              : t->opt == DHS_ADAGRAD ? (ext ? launch_seg_adagrad_ext : launch_seg_adagrad)
              : t->opt == DHS_ADAM ? (ext ? launch_seg_adam_ext : launch_seg_adam)
                                   : (ext ? launch_seg_rowwise_ext : launch_seg_rowwise);
    e = fn(G, NV, t->sm_count, sk, sv, n, grad, nb, t->dim, rowspace(t), oa, part_head, part_tail,
           seg_chunk(n), chunk_ctr, owners, owner_ctr, t->st, bagpos, mult, mean,
           DHS_SEG_RUN_TABLE_NARROW ? rt : RunTable{}, s);
  }
  t->n_launches++;
  if (e != cudaSuccess) cudaGetLastError();
  return e == cudaSuccess ? DHS_OK : DHS_ERR_CUDA;
}

// The arrival table of a backward of n ids (its key and ctr arrays are
// cleared by the probe kernel: the first 2 * (mask + 1) words of b_runs).
RunTable run_table(dhs_table* t, long long n) {
  RunTable rt;
  const long long cap = std::min(run_table_cap((n + seg_chunk(n) - 1) / seg_chunk(n)), t->ws_run_cap);
  unsigned* w = (unsigned*)t->b_runs.p;
  rt.key = w;
  rt.ctr = w + cap;
  rt.c0 = w + 2 * cap;
  rt.c1 = w + 3 * cap;
  rt.mask = (unsigned)(cap - 1);
  rt.max_pieces = kSegFinishPieces;
  if (!DHS_SEG_RUN_TABLE) rt.key = nullptr;
  return rt;
}

// The counters of the current backward (zero when it starts).
unsigned* hist_words(dhs_table* t) { return (unsigned*)t->b_hist.p + (size_t)t->hist_sel * kSortZeroWords; }

dhs_status dispatch_seg(dhs_table* t, const unsigned* sk, const unsigned* sv, long long n,
                        const float* grad, long long nb, const OptArgs& oa, bool ext, bool mean, unsigned* ctr,
                        cudaStream_t s) {
  return launch_seg(t, sk, sv, n, grad, nb, oa, (double*)t->b_ph.p, (double*)t->b_pt.p,
                    ctr + kSegChunkCtrWord, (unsigned*)t->b_owners.p,
                    ctr + kSegOwnerCtrWord, ext ? (const unsigned*)t->b_bagpos.p : nullptr,
                    ext ? (const double*)t->b_mult.p : nullptr, mean, run_table(t, n), s);
}

// offset assignment + row init for the new keys of an insert call
dhs_status launch_assign(dhs_table* t, const long long* keys, long long n, cudaStream_t s) {
  const long long nwords = (n + 31) / 32;
  const long long ngroups = (n + kGroupPositions - 1) / kGroupPositions;
  launch_k(fwd_mark_kernel, (unsigned)ngroups, kGroupThreads, 0, s, 
      t->slots, (unsigned*)t->b_nbm.p, (unsigned*)t->b_fbm.p, (unsigned*)t->b_gcnt.p,
      (unsigned*)t->b_gpref.p, (const unsigned*)t->b_slotpos.p, nwords, ngroups, hooks(t), t->st);
  t->n_launches += 2;
  DHS_TRY(last_launch());
  launch_k(fwd_assign_kernel, (unsigned)ngroups, kGroupThreads, 0, s, 
      t->slots, rowspace(t), t->dim, keys, (const unsigned*)t->b_fbm.p, (const unsigned*)t->b_gpref.p,
      (const unsigned*)t->b_slotpos.p, nwords, ngroups, hooks(t), t->st);
  return last_launch();
}

int state_floats(int opt, int dim) {
  switch (opt) {
    case DHS_SGD: return 0;
    case DHS_ADAGRAD: return dim;
    case DHS_ADAM: return 2 * dim;
    case DHS_ADAGRAD_ROWWISE: return 4;  // accumulator + 3 pad floats (16-byte rows)
  }
  return -1;
}

}  // namespace

extern "C" {

const char* dhs_status_str(dhs_status s) {
  switch (s) {
    case DHS_OK: return "ok";
    case DHS_ERR_INVALID_ARG: return "invalid argument";
    case DHS_ERR_OOM: return "out of device memory";
    case DHS_ERR_CUDA: return "CUDA error";
    case DHS_ERR_TABLE_FULL: return "table full";
    case DHS_ERR_NOT_FOUND: return "key not found";
    case DHS_ERR_UNSUPPORTED: return "unsupported";
    case DHS_ERR_INTERNAL: return "internal wait bound exceeded";
  }
  return "unknown status";
}

dhs_status dhs_pack_keys(const int32_t* d_table_ids, const int64_t* d_ids, int64_t n,
                         int64_t* d_keys_out, dhs_stream stream) {
  if (n < 0 || (n > 0 && (!d_table_ids || !d_ids || !d_keys_out))) return DHS_ERR_INVALID_ARG;
  if (n == 0) return DHS_OK;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long grid = std::min<long long>((n + 255) / 256, (long long)sms * 8);
  launch_k(pack_keys_kernel, (unsigned)grid, 256, 0, (cudaStream_t)stream, 
      d_table_ids, (const long long*)d_ids, n, (long long*)d_keys_out);
  return last_launch();
}

dhs_status ht_create_ex(int32_t dim, dhs_optimizer opt, dhs_row_dtype weights, int64_t block_rows,
                        int64_t max_rows, const dhs_opt_params* params, const dhs_allocator* alloc,
                        dhs_table** out) {
  if (!out) return DHS_ERR_INVALID_ARG;
  *out = nullptr;
  if (dim < 4 || dim > 512 || dim % 4) return DHS_ERR_INVALID_ARG;
  if (weights != DHS_ROWS_F32 && weights != DHS_ROWS_BF16) return DHS_ERR_INVALID_ARG;
  // bf16 rows: 8 weights per 16-byte unit, warp segment kernel (dim >= 32)
  if (weights == DHS_ROWS_BF16 && (dim % 8 || dim < DHS_SEGW_MIN_DIM)) return DHS_ERR_UNSUPPORTED;
  if (state_floats(opt, dim) < 0) return DHS_ERR_INVALID_ARG;
  if (block_rows == 0) block_rows = kDefaultBlockRows;
  if (block_rows < 1 || (block_rows & (block_rows - 1)) || block_rows > (1ll << 30))
    return DHS_ERR_INVALID_ARG;
  if (max_rows == 0) max_rows = kDefaultMaxRows;
  if (max_rows < 1 || max_rows > kMaxRowsLimit) return DHS_ERR_INVALID_ARG;
  if (alloc && (!alloc->alloc || !alloc->free)) return DHS_ERR_INVALID_ARG;
  if (params && !(params->eps >= 0.f && params->beta1 >= 0.f && params->beta1 < 1.f &&
                  params->beta2 >= 0.f && params->beta2 < 1.f))
    return DHS_ERR_INVALID_ARG;

  dhs_table* t = new (std::nothrow) dhs_table();
  if (!t) return DHS_ERR_OOM;
  if (cudaGetDevice(&t->device) != cudaSuccess) {
    cudaGetLastError();
    delete t;
    return DHS_ERR_CUDA;
  }
  cudaDeviceGetAttribute(&t->sm_count, cudaDevAttrMultiProcessorCount, t->device);
  t->dim = dim;
  t->opt = opt;
  t->wbf16 = weights == DHS_ROWS_BF16;
  t->wfl = t->wbf16 ? dim / 2 : dim;
  t->stride = t->wfl + state_floats(opt, dim);
  if (params) {
    t->eps = params->eps;
    t->b1 = params->beta1;
    t->b2 = params->beta2;
  }
  t->block_rows = block_rows;
  t->log2_br = log2_exact(block_rows);
  t->max_rows = max_rows;
  t->max_blocks = (max_rows + block_rows - 1) / block_rows;
  if (alloc) {
    t->alloc = *alloc;
    t->custom_alloc = true;
  }
  cudaStream_t s = nullptr;
  dhs_status rc = DHS_OK;
  if (!t->custom_alloc) {
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = t->device;
    if (cudaMemPoolCreate(&t->pool, &props) != cudaSuccess) {
      cudaGetLastError();
      delete t;
      return DHS_ERR_CUDA;
    }
    unsigned long long keep = ~0ull;  // never hand freed memory back to the driver
    cudaMemPoolSetAttribute(t->pool, cudaMemPoolAttrReleaseThreshold, &keep);
  }
  t->st = (DevState*)dalloc(t, sizeof(DevState), s);
  t->blocks_d = (float**)dalloc(t, sizeof(float*) * t->max_blocks, s);
  if (!t->st || !t->blocks_d) rc = DHS_ERR_OOM;
  if (rc == DHS_OK && cudaMemsetAsync(t->st, 0, sizeof(DevState), s) != cudaSuccess) rc = DHS_ERR_CUDA;
  if (rc == DHS_OK && cudaMemsetAsync(t->blocks_d, 0, sizeof(float*) * t->max_blocks, s) != cudaSuccess)
    rc = DHS_ERR_CUDA;
  for (int i = 0; rc == DHS_OK && i < kSnapRing; ++i) {
    if (cudaEventCreateWithFlags(&t->snaps[i].ev, cudaEventDisableTiming) != cudaSuccess ||
        cudaHostAlloc((void**)&t->snaps[i].pinned, 3 * sizeof(unsigned long long), cudaHostAllocMapped) !=
            cudaSuccess ||
        cudaHostGetDevicePointer((void**)&t->snaps[i].pinned_dev, t->snaps[i].pinned, 0) != cudaSuccess)
      rc = DHS_ERR_CUDA;
  }
  if (rc == DHS_OK) rc = grow_map(t, kInitialSlots, s);
  if (rc == DHS_OK && cudaStreamSynchronize(s) != cudaSuccess) rc = DHS_ERR_CUDA;
  if (rc != DHS_OK) {
    cudaGetLastError();
    ht_destroy(t);
    return rc;
  }
  t->last_stream = s;
  *out = t;
  return DHS_OK;
}

dhs_status ht_create(int32_t dim, dhs_optimizer opt, int64_t block_rows, int64_t max_rows,
                     const dhs_opt_params* params, const dhs_allocator* alloc, dhs_table** out) {
  return ht_create_ex(dim, opt, DHS_ROWS_F32, block_rows, max_rows, params, alloc, out);
}

dhs_status ht_destroy(dhs_table* t) {
  if (!t) return DHS_OK;
  DeviceGuard g(t->device);
  cudaStream_t s = t->last_stream;
  cudaStreamSynchronize(s);
  cudaDeviceSynchronize();
  s = nullptr;
  for (float* b : t->blocks_h) dfree(t, b, (size_t)t->block_rows * t->stride * sizeof(float), s);
  t->blocks_h.clear();
  dfree(t, t->slots, t->nslots * sizeof(Slot), s);
  dfree(t, t->blocks_d, sizeof(float*) * t->max_blocks, s);
  dfree(t, t->st, sizeof(DevState), s);
  if (t->cnt) dfree(t, t->cnt, t->nslots * 4, s);
  if (t->stamp) dfree(t, t->stamp, t->nslots * 4, s);
  if (t->free_bm) dfree(t, t->free_bm, (size_t)t->free_words * 4, s);
  if (t->free_list) dfree(t, t->free_list, (size_t)t->free_list_cap * 4, s);
  Buf* bufs[] = {&t->b_fcnt, &t->b_freed, &t->b_nbm, &t->b_fbm, &t->b_gcnt, &t->b_gpref, &t->b_slotpos, &t->b_ka, &t->b_va,
                 &t->b_kb, &t->b_vb, &t->b_hist, &t->b_totals, &t->b_ph, &t->b_pt, &t->b_owners,
                 &t->b_cplan, &t->b_slots, &t->b_refs, &t->b_bagpos, &t->b_mult, &t->b_runs, &t->b_shard,
                 &t->b_reckey};
  for (Buf* b : bufs) bfree(t, *b, s);
  cudaStreamSynchronize(s);
  for (auto& sn : t->snaps) {
    if (sn.ev) cudaEventDestroy(sn.ev);
    if (sn.pinned) cudaFreeHost(sn.pinned);
  }
  if (t->pool) cudaMemPoolDestroy(t->pool);
  for (auto& r : t->recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (cudaEvent_t e : t->ev_pool) cudaEventDestroy(e);
  cudaGetLastError();
  delete t;
  return DHS_OK;
}

dhs_status ht_reserve(dhs_table* t, int64_t n_keys, dhs_stream stream) {
  DHS_TRY(check_table(t));
  if (n_keys < 0) return DHS_ERR_INVALID_ARG;
  t->rec_n = -1;
  DeviceGuard g(t->device);
  cudaStream_t s = (cudaStream_t)stream;
  t->last_stream = s;
  if ((double)n_keys > kMaxLoad * (double)t->nslots)
    DHS_TRY(grow_map(t, (unsigned long long)std::ceil((double)n_keys / kMaxLoad), s));
  const long long rows = std::min<long long>(n_keys, t->max_rows);
  while ((long long)t->blocks_h.size() * t->block_rows < rows) {
    const size_t bytes = (size_t)t->block_rows * t->stride * sizeof(float);
    float* b = (float*)dalloc(t, bytes, s);
    if (!b) return DHS_ERR_OOM;
    t->blocks_h.push_back(b);
    set_block_kernel<<<1, 1, 0, s>>>(t->blocks_d, (long long)t->blocks_h.size() - 1, b, t->st,
                                     (unsigned long long)t->blocks_h.size());
    t->n_launches++;
    DHS_TRY(last_launch());
  }
  return DHS_OK;
}

dhs_status ht_lookup_or_insert(dhs_table* t, const int64_t* d_keys, int64_t n,
                               int64_t* d_offsets_out, dhs_stream stream) {
  DHS_TRY(check_table(t));
  if (n < 0 || n >= (1ll << 31) || (n > 0 && (!d_keys || !d_offsets_out))) return DHS_ERR_INVALID_ARG;
  t->rec_n = -1;
  if (n == 0) {
    t->step++;  // every insert call is a step of the access stamps
    return DHS_OK;
  }
  DeviceGuard g(t->device);
  cudaStream_t s = (cudaStream_t)stream;
  t->last_stream = s;
  DHS_TRY(ensure_capacity(t, n, s));
  DHS_TRY(ensure_ws(t, n, s));
  t->step++;
  {
    PhaseScope ph(t, PH_LOOKUP_INSERT, s);
    launch_k(fwd_probe_offsets_kernel, (unsigned)((n + kFwdThreads - 1) / kFwdThreads), kFwdThreads, 0, s, 
        idmap(t), (const long long*)d_keys, n, (long long*)d_offsets_out, (unsigned*)t->b_nbm.p,
        (unsigned*)t->b_slotpos.p, (long long*)nullptr, hooks(t), t->st);
    t->n_launches += 2;
    DHS_TRY(last_launch());
    DHS_TRY(launch_assign(t, (const long long*)d_keys, n, s));
    const long long grid = std::min<long long>((n + 255) / 256, (long long)t->sm_count * 8);
    launch_k(fwd_fixup_kernel, (unsigned)grid, 256, 0, s, t->slots, (long long*)d_offsets_out, n);
    DHS_TRY(last_launch());
  }
  t->rows_ub += n;
  t->keys_ub += n;
  t->cum_n += n;
  t->n_insert_calls++;
  record_snapshot(t, s);
  return DHS_OK;
}

dhs_status ht_lookup(dhs_table* t, const int64_t* d_keys, int64_t n, int64_t* d_offsets_out,
                     dhs_stream stream) {
  DHS_TRY(check_table(t));
  if (n < 0 || (n > 0 && (!d_keys || !d_offsets_out))) return DHS_ERR_INVALID_ARG;
  if (n == 0) return DHS_OK;
  DeviceGuard g(t->device);
  cudaStream_t s = (cudaStream_t)stream;
  t->last_stream = s;
  const long long grid = std::min<long long>((n + 255) / 256, (long long)t->sm_count * 16);
  launch_k(lookup_kernel, (unsigned)grid, 256, 0, s, idmap(t), (const long long*)d_keys, n, (long long*)d_offsets_out);
  t->n_launches++;
  return last_launch();
}

dhs_status embbag_forward_ex(dhs_table* t, const int64_t* d_keys, int64_t n_keys,
                             const int64_t* d_bag_offsets, int64_t n_bags, const float* d_per_sample_weights,
                             dhs_pool_mode mode, float* d_pooled_out, dhs_stream stream) {
  DHS_TRY(check_table(t));
  if (n_keys < 0 || n_keys >= (1ll << 31) || n_bags < 0 || n_bags >= (1ll << 31))
    return DHS_ERR_INVALID_ARG;
  if (mode != DHS_POOL_SUM && mode != DHS_POOL_MEAN) return DHS_ERR_INVALID_ARG;
  if (mode == DHS_POOL_MEAN && d_per_sample_weights) return DHS_ERR_INVALID_ARG;
  const bool mean = mode == DHS_POOL_MEAN;
  const float* psw = n_keys > 0 ? d_per_sample_weights : nullptr;
  t->rec_n = -1;
  if (n_bags == 0) {
    if (n_keys != 0) return DHS_ERR_INVALID_ARG;
    t->step++;  // every insert call is a step of the access stamps
    return DHS_OK;
  }
  if (!d_bag_offsets || !d_pooled_out || (n_keys > 0 && !d_keys)) return DHS_ERR_INVALID_ARG;
  if ((uintptr_t)d_pooled_out % 16) return DHS_ERR_INVALID_ARG;
  DeviceGuard g(t->device);
  cudaStream_t s = (cudaStream_t)stream;
  t->last_stream = s;
  if (n_keys > 0) DHS_TRY(ensure_capacity(t, n_keys, s));
  DHS_TRY(ensure_ws(t, n_keys, s));
  t->step++;
  // admission and eviction need the split forward (the probe counts and
  // stamps, the assignment decides which keys get a row before the gather)
  if (n_keys > 0 && (n_keys >= (long long)DHS_POOL_SPLIT_LEN * n_bags || has_hooks(t))) {
    // long bags: probe every id (a thread per id), assign and write the new
    // keys' rows, then gather every row from the table
    {
      PhaseScope ph(t, PH_FWD_PROBE, s);
      launch_k(fwd_probe_offsets_kernel, (unsigned)((n_keys + kFwdThreads - 1) / kFwdThreads), kFwdThreads, 0, s, 
          idmap(t), (const long long*)d_keys, n_keys, (long long*)t->b_refs.p, (unsigned*)t->b_nbm.p,
          (unsigned*)t->b_slotpos.p, (long long*)t->b_reckey.p, hooks(t), t->st);
      t->n_launches++;
      DHS_TRY(last_launch());
    }
    {
      PhaseScope ph(t, PH_FWD_ASSIGN, s);
      DHS_TRY(launch_assign(t, (const long long*)d_keys, n_keys, s));
    }
    {
      PhaseScope ph(t, PH_FWD_POOL, s);
      const int wd = t->wbf16 ? t->dim / 2 : t->dim;
      const int G = pick_group(wd), NV = pick_nv(wd, G);
      const cudaError_t e = (t->wbf16 ? launch_pool_refs_bf16 : launch_pool_refs)(
          G, NV, t->sm_count, rowspace(t), t->dim, t->slots, (long long*)t->b_refs.p, n_keys,
          (const long long*)d_bag_offsets, n_bags, psw, mean, d_pooled_out, t->st, s);
      t->n_launches++;
      if (e != cudaSuccess) {
        cudaGetLastError();
        return DHS_ERR_CUDA;
      }
    }
    t->rec_n = n_keys;  // keys and rows of every position recorded
  } else {
    {
      PhaseScope ph(t, PH_FWD_POOL, s);
      DHS_TRY(dispatch_pool(t, (const long long*)d_keys, n_keys, (const long long*)d_bag_offsets,
                            n_bags, psw, mean, d_pooled_out, s));
    }
    if (n_keys > 0) {
      PhaseScope ph(t, PH_FWD_ASSIGN, s);
      DHS_TRY(launch_assign(t, (const long long*)d_keys, n_keys, s));
    }
  }
  t->n_insert_calls++;
  if (n_keys > 0) {
    t->rows_ub += n_keys;
    t->keys_ub += n_keys;
    t->cum_n += n_keys;
    record_snapshot(t, s);
  }
  return DHS_OK;
}

dhs_status embbag_forward(dhs_table* t, const int64_t* d_keys, int64_t n_keys,
                          const int64_t* d_bag_offsets, int64_t n_bags, float* d_pooled_out,
                          dhs_stream stream) {
  return embbag_forward_ex(t, d_keys, n_keys, d_bag_offsets, n_bags, nullptr, DHS_POOL_SUM, d_pooled_out, stream);
}

dhs_status embbag_backward_update_ex(dhs_table* t, const int64_t* d_keys, int64_t n_keys,
                                     const int64_t* d_bag_offsets, int64_t n_bags,
                                     const float* d_per_sample_weights, dhs_pool_mode mode,
                                     const float* d_grad, float lr, dhs_stream stream) {
  DHS_TRY(check_table(t));
  if (n_keys < 0 || n_keys >= (1ll << 31) || n_bags < 0 || n_bags >= (1ll << 31))
    return DHS_ERR_INVALID_ARG;
  if (mode != DHS_POOL_SUM && mode != DHS_POOL_MEAN && mode != DHS_POOL_DIVIDE) return DHS_ERR_INVALID_ARG;
  if (mode == DHS_POOL_MEAN && d_per_sample_weights) return DHS_ERR_INVALID_ARG;
  if (mode == DHS_POOL_DIVIDE && n_keys > 0 && !d_per_sample_weights) return DHS_ERR_INVALID_ARG;
  // mean pooling divides each id's term by its bag's length (DHS_POOL_DIVIDE:
  // by the per-id value given)
  const bool mean = mode == DHS_POOL_MEAN || mode == DHS_POOL_DIVIDE;
  const float* psw = n_keys > 0 ? d_per_sample_weights : nullptr;
  const bool ext = psw != nullptr || mean;
  if (n_bags == 0 && n_keys != 0) return DHS_ERR_INVALID_ARG;
  if (n_bags > 0 && (!d_bag_offsets || !d_grad)) return DHS_ERR_INVALID_ARG;
  if ((uintptr_t)d_grad % 16) return DHS_ERR_INVALID_ARG;
  if (n_keys > 0 && !d_keys) return DHS_ERR_INVALID_ARG;
  if (!std::isfinite(lr)) return DHS_ERR_INVALID_ARG;
  DeviceGuard g(t->device);
  cudaStream_t s = (cudaStream_t)stream;
  t->last_stream = s;
  t->adam_t += 1;
  t->bwd_n += n_keys;
  if (n_keys == 0) return DHS_OK;
  DHS_TRY(ensure_ws(t, n_keys, s));
  if (ext) DHS_TRY(ensure_ws_ext(t, s));

  // rows of the table are < rows_ub; rows_ub itself marks a missing key
  refresh_ub(t, false);
  const unsigned sentinel = (unsigned)t->rows_ub;
  int bits = 0;
  while (bits < 32 && (1ull << bits) <= (unsigned long long)sentinel) ++bits;
  const int passes = std::min(kRadixMaxPasses, std::max(1, (bits + 7) / 8));

  unsigned* ka = (unsigned*)t->b_ka.p;
  unsigned* va = (unsigned*)t->b_va.p;
  unsigned* kb = (unsigned*)t->b_kb.p;
  unsigned* vb = (unsigned*)t->b_vb.p;
  unsigned* const ctr = hist_words(t);  // this backward's counters
  {
    PhaseScope ph(t, PH_BWD_PROBE, s);
    const int bpc = bwd_probe_bags(n_keys, n_bags);
    const long long ntiles = (n_keys + kRadixTile - 1) / kRadixTile;
    // the last insert call was a split forward over as many positions: its
    // record of keys and rows stands in for the probe where the keys agree
    const bool rec = DHS_BWD_RECORD && t->rec_n == n_keys;
    // the counters this backward accumulates into are zero (cleared by the
    // previous backward's probe, or at allocation); this probe clears the
    // other area for the next one
    unsigned* next_hist = (unsigned*)t->b_hist.p + (size_t)(1 - t->hist_sel) * kSortZeroWords;
    const long long zero_runs = 2 * ((long long)run_table(t, n_keys).mask + 1);
    // one resident wave of blocks, each warp taking chunks of bags in turn:
    // each block flushes its digit counts with one atomic per nonzero bin,
    // so fewer blocks mean fewer atomics on the shared counters
    const int resident = resident_blocks(ext ? bwd_probe_kernel<true> : bwd_probe_kernel<false>, 256, 0,
                                         t->sm_count);
    const long long warps = (n_bags + bpc - 1) / bpc;
    const long long grid = grid_for((warps + 7) / 8, resident);
    (void)launch_k(ext ? bwd_probe_kernel<true> : bwd_probe_kernel<false>, (unsigned)grid, 256, 0, s, idmap(t),
                   (const long long*)d_keys, n_keys, (const long long*)d_bag_offsets, n_bags, ka, va, sentinel, ctr,
                   passes, (unsigned long long*)t->b_totals.p, ntiles * kRadixBins, (unsigned*)t->b_runs.p,
                   zero_runs, next_hist, (long long)kSortZeroWords, bpc, psw, mean, (unsigned*)t->b_bagpos.p,
                   (double*)t->b_mult.p, rec ? (const long long*)t->b_reckey.p : nullptr,
                   rec ? (const long long*)t->b_refs.p : nullptr, t->st);
    t->n_launches++;
    DHS_TRY(last_launch());
    t->hist_sel ^= 1;  // the next backward uses the area this probe cleared
  }
  {
    PhaseScope ph(t, PH_BWD_SORT, s);
    const long long ntiles = (n_keys + kRadixTile - 1) / kRadixTile;
    unsigned* hist = ctr;
    unsigned* tile_ctr = hist + kRadixMaxPasses * kRadixBins;
    unsigned long long* status = (unsigned long long*)t->b_totals.p;
    for (int p = 0; p < passes; ++p) {
      const long long words = ntiles * kRadixBins;
      launch_k(radix_onesweep_kernel, (unsigned)ntiles, kRadixThreads, 0, s, 
          ka, va, kb, vb, n_keys, 8 * p, hist + p * kRadixBins, status + (long long)p * words, tile_ctr + p,
          status + (long long)(p + 1) * words, p + 1 < passes ? words : 0, t->st);
      t->n_launches++;
      DHS_TRY(last_launch());
      std::swap(ka, kb);
      std::swap(va, vb);
    }
  }
  {
    OptArgs oa;
    oa.opt = t->opt;
    oa.lr = lr;
    oa.eps = t->eps;
    oa.b1 = t->b1;
    oa.b2 = t->b2;
    oa.c1 = (float)(1.0 - (double)t->b1);
    oa.c2 = (float)(1.0 - (double)t->b2);
    oa.bc1 = (float)(1.0 - std::pow((double)t->b1, (double)t->adam_t));
    oa.bc2 = (float)(1.0 - std::pow((double)t->b2, (double)t->adam_t));
    {
      PhaseScope ph(t, PH_BWD_SEG, s);
      DHS_TRY(dispatch_seg(t, ka, va, n_keys, d_grad, n_bags, oa, ext, mean, ctr, s));
    }
    PhaseScope ph(t, PH_BWD_COMBINE, s);
    const int pstride = seg_nv(t->dim) * seg_group(t->dim) * 4;
    DHS_TRY(launch_combine(t, ka, n_keys, oa, (const double*)t->b_ph.p, (const double*)t->b_pt.p,
                           seg_chunk(n_keys), pstride, (const unsigned*)t->b_owners.p,
                           ctr,
                           combine_plan((unsigned*)t->b_cplan.p, (double*)t->b_slots.p, t->ws_chunks, ctr),
                           s));
  }
  return DHS_OK;
}

dhs_status embbag_backward_update(dhs_table* t, const int64_t* d_keys, int64_t n_keys,
                                  const int64_t* d_bag_offsets, int64_t n_bags,
                                  const float* d_grad, float lr, dhs_stream stream) {
  return embbag_backward_update_ex(t, d_keys, n_keys, d_bag_offsets, n_bags, nullptr, DHS_POOL_SUM, d_grad, lr,
                                   stream);
}

dhs_status ht_get_rows(dhs_table* t, const int64_t* d_keys, int64_t n, float* d_rows_out,
                       dhs_stream stream) {
  DHS_TRY(check_table(t));
  if (n < 0 || (n > 0 && (!d_keys || !d_rows_out))) return DHS_ERR_INVALID_ARG;
  if (n == 0) return DHS_OK;
  DeviceGuard g(t->device);
  cudaStream_t s = (cudaStream_t)stream;
  t->last_stream = s;
  const long long grid = std::min<long long>((n + 7) / 8, (long long)t->sm_count * 16);
  launch_k(get_rows_kernel, (unsigned)grid, 256, 0, s, idmap(t), rowspace(t), t->dim, export_stride(t),
                                                 (const long long*)d_keys, n, d_rows_out);
  t->n_launches++;
  return last_launch();
}

dhs_status ht_set_hooks(dhs_table* t, int64_t admit_threshold, int track_access) {
  DHS_TRY(check_table(t));
  if (admit_threshold < 0 || admit_threshold > 0x7fffffff) return DHS_ERR_INVALID_ARG;
  if (t->step > 0 || t->rows_ub > 0 || t->has_hooks_set) return DHS_ERR_INVALID_ARG;  // before the first insert, once
  DeviceGuard g(t->device);
  cudaStream_t s = t->last_stream;
  t->admit = (unsigned)std::max<int64_t>(1, admit_threshold);
  t->track = track_access != 0;
  t->has_hooks_set = true;
  if (t->admit > 1) {
    t->cnt = (unsigned*)dalloc(t, t->nslots * 4, s);
    if (!t->cnt) return DHS_ERR_OOM;
    DHS_CUDA(cudaMemsetAsync(t->cnt, 0, t->nslots * 4, s));
  }
  if (t->track) {
    t->stamp = (unsigned*)dalloc(t, t->nslots * 4, s);
    if (!t->stamp) return DHS_ERR_OOM;
    DHS_CUDA(cudaMemsetAsync(t->stamp, 0, t->nslots * 4, s));
  }
  DHS_CUDA(cudaMemsetAsync(&t->st->keys_used, 0, sizeof(unsigned long long), s));
  return DHS_OK;
}

dhs_status ht_evict(dhs_table* t, int64_t max_idle, int64_t* n_freed, dhs_stream stream) {
  DHS_TRY(check_table(t));
  if (!t->track || max_idle < 0 || !n_freed) return DHS_ERR_INVALID_ARG;
  t->rec_n = -1;  // evicted keys lose their rows
  DeviceGuard g(t->device);
  cudaStream_t s = (cudaStream_t)stream;
  t->last_stream = s;
  *n_freed = 0;
  const long long keep_from = t->step - max_idle;  // keys last seen before this step go
  if (keep_from <= 1) return DHS_OK;                // every stamp is >= 1
  DHS_CUDA(cudaStreamSynchronize(s));
  unsigned long long rows = 0;
  DHS_CUDA(cudaMemcpy(&rows, &t->st->row_count, sizeof(rows), cudaMemcpyDeviceToHost));
  // the free-row bitmap covers every row; the list can hold them all
  const long long words = (long long)((rows + 31) / 32);
  if (words > t->free_words) {
    const long long nw = std::max<long long>(words, t->free_words * 2);
    unsigned* nb = (unsigned*)dalloc(t, (size_t)nw * 4, s);
    if (!nb) return DHS_ERR_OOM;
    DHS_CUDA(cudaMemsetAsync(nb, 0, (size_t)nw * 4, s));
    if (t->free_bm) {
      DHS_CUDA(cudaMemcpyAsync(nb, t->free_bm, (size_t)t->free_words * 4, cudaMemcpyDeviceToDevice, s));
      dfree(t, t->free_bm, (size_t)t->free_words * 4, s);
    }
    t->free_bm = nb;
    t->free_words = nw;
  }
  if ((long long)rows > t->free_list_cap) {
    const long long cap = std::max<long long>((long long)rows, t->free_list_cap * 2);
    unsigned* nl = (unsigned*)dalloc(t, (size_t)cap * 4, s);
    if (!nl) return DHS_ERR_OOM;
    if (t->free_list) dfree(t, t->free_list, (size_t)t->free_list_cap * 4, s);
    t->free_list = nl;
    t->free_list_cap = cap;
  }
  const long long nblocks = std::max<long long>(1, (words + kFreeWords - 1) / kFreeWords);
  DHS_TRY(bget(t, t->b_fcnt, (size_t)nblocks * 4, s));
  DHS_TRY(bget(t, t->b_freed, sizeof(unsigned long long), s));
  DHS_CUDA(cudaMemsetAsync(t->b_freed.p, 0, sizeof(unsigned long long), s));
  const int thr = 256;
  const long long g1 = std::min<long long>((long long)((t->nslots + thr - 1) / thr), (long long)t->sm_count * 16);
  evict_kernel<<<(unsigned)g1, thr, 0, s>>>(t->slots, t->nslots, t->stamp, (unsigned)keep_from, t->free_bm,
                                            (unsigned long long*)t->b_freed.p);
  free_count_kernel<<<(unsigned)nblocks, kFreeThreads, 0, s>>>(t->free_bm, words, (unsigned*)t->b_fcnt.p,
                                                                nblocks, t->st);
  free_scatter_kernel<<<(unsigned)nblocks, kFreeThreads, 0, s>>>(t->free_bm, words, (const unsigned*)t->b_fcnt.p,
                                                                  t->free_list);
  t->n_launches += 3;
  DHS_TRY(last_launch());
  unsigned long long freed = 0;
  DHS_CUDA(cudaMemcpyAsync(&freed, t->b_freed.p, sizeof(freed), cudaMemcpyDeviceToHost, s));
  DHS_CUDA(cudaStreamSynchronize(s));
  *n_freed = (int64_t)freed;
  return DHS_OK;
}

dhs_status ht_live_rows(dhs_table* t, int64_t* n_live) {
  DHS_TRY(check_table(t));
  if (!n_live) return DHS_ERR_INVALID_ARG;
  const dhs_status rc = ht_sync(t);
  if (rc == DHS_ERR_CUDA) return rc;
  DeviceGuard g(t->device);
  DevState h;
  DHS_CUDA(cudaMemcpy(&h, t->st, sizeof(h), cudaMemcpyDeviceToHost));
  *n_live = (int64_t)(h.row_count - (h.free_count - h.free_head));
  return rc;
}

int64_t ht_row_stride(const dhs_table* t) { return t ? export_stride(t) : -1; }

dhs_status ht_sync(dhs_table* t) {
  DHS_TRY(check_table(t));
  DeviceGuard g(t->device);
  DHS_CUDA(cudaStreamSynchronize(t->last_stream));
  DHS_CUDA(cudaDeviceSynchronize());
  unsigned err = 0;
  DHS_CUDA(cudaMemcpy(&err, &t->st->err, sizeof(unsigned), cudaMemcpyDeviceToHost));
  if (err) {
    const unsigned zero = 0;
    DHS_CUDA(cudaMemcpy(&t->st->err, &zero, sizeof(unsigned), cudaMemcpyHostToDevice));
  }
  return (dhs_status)err;
}

dhs_status ht_size(dhs_table* t, int64_t* n_rows) {
  DHS_TRY(check_table(t));
  if (!n_rows) return DHS_ERR_INVALID_ARG;
  const dhs_status rc = ht_sync(t);
  if (rc == DHS_ERR_CUDA) return rc;
  DeviceGuard g(t->device);
  unsigned long long r = 0;
  DHS_CUDA(cudaMemcpy(&r, &t->st->row_count, sizeof(r), cudaMemcpyDeviceToHost));
  *n_rows = (int64_t)r;
  t->rows_ub = (long long)r;
  return rc;
}

dhs_status ht_counters(dhs_table* t, int64_t out[14]) {
  DHS_TRY(check_table(t));
  if (!out) return DHS_ERR_INVALID_ARG;
  DeviceGuard g(t->device);
  DHS_CUDA(cudaStreamSynchronize(t->last_stream));
  DHS_CUDA(cudaDeviceSynchronize());
  DevState h;
  DHS_CUDA(cudaMemcpy(&h, t->st, sizeof(h), cudaMemcpyDeviceToHost));
  out[0] = (int64_t)h.row_count;
  out[1] = (int64_t)h.sum_new;
  out[2] = (int64_t)h.sum_unique;
  out[3] = t->n_insert_calls;
  out[4] = t->adam_t;
  out[5] = (int64_t)t->nslots;
  out[6] = (int64_t)t->blocks_h.size();
  out[7] = t->n_rehash;
  out[8] = t->n_launches;
  out[9] = (int64_t)h.m_last;
  out[10] = t->n_host_waits;
  out[11] = t->host_wait_ns;
  out[12] = t->n_allocs;
  out[13] = t->alloc_ns;
  return DHS_OK;
}

dhs_status ht_export(dhs_table* t, int64_t* h_keys, float* h_rows) {
  DHS_TRY(check_table(t));
  int64_t rows = 0;
  const dhs_status rc = ht_size(t, &rows);
  if (rc == DHS_ERR_CUDA) return rc;
  DeviceGuard g(t->device);
  cudaStream_t s = t->last_stream;
  if (h_keys && rows > 0) {
    long long* kb = (long long*)dalloc(t, sizeof(long long) * rows, s);
    if (!kb) return DHS_ERR_OOM;
    const long long grid = std::min<long long>((long long)((t->nslots + 255) / 256), (long long)t->sm_count * 16);
    DHS_CUDA(cudaMemsetAsync(kb, 0xff, sizeof(long long) * rows, s));  // a free (evicted) row has key -1
    keys_by_row_kernel<<<(unsigned)grid, 256, 0, s>>>(t->slots, t->nslots, kb, (unsigned long long)rows);
    dhs_status lr = last_launch();
    if (lr == DHS_OK && cudaMemcpyAsync(h_keys, kb, sizeof(long long) * rows, cudaMemcpyDeviceToHost, s) != cudaSuccess)
      lr = DHS_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) lr = DHS_ERR_CUDA;
    dfree(t, kb, sizeof(long long) * rows, s);
    cudaStreamSynchronize(s);
    DHS_TRY(lr);
  }
  if (h_rows && !t->wbf16) {
    for (long long r0 = 0; r0 < rows; r0 += t->block_rows) {
      const long long cnt = std::min<long long>(t->block_rows, rows - r0);
      DHS_CUDA(cudaMemcpy(h_rows + r0 * t->stride, t->blocks_h[r0 >> t->log2_br],
                          sizeof(float) * cnt * t->stride, cudaMemcpyDeviceToHost));
    }
  } else if (h_rows) {
    // bf16 weights: each block's raw rows, widened on the host to the fp32
    // export layout (dim weights, then the state)
    const int es = export_stride(t);
    std::vector<float> raw;
    for (long long r0 = 0; r0 < rows; r0 += t->block_rows) {
      const long long cnt = std::min<long long>(t->block_rows, rows - r0);
      raw.resize((size_t)cnt * t->stride);
      DHS_CUDA(cudaMemcpy(raw.data(), t->blocks_h[r0 >> t->log2_br], sizeof(float) * cnt * t->stride,
                          cudaMemcpyDeviceToHost));
      for (long long r = 0; r < cnt; ++r) {
        const float* src = raw.data() + r * t->stride;
        float* dst = h_rows + (r0 + r) * es;
        const uint16_t* w = reinterpret_cast<const uint16_t*>(src);
        for (int j = 0; j < t->dim; ++j) {
          const uint32_t u = (uint32_t)w[j] << 16;
          std::memcpy(dst + j, &u, 4);
        }
        std::memcpy(dst + t->dim, src + t->wfl, sizeof(float) * (t->stride - t->wfl));
      }
    }
  }
  return rc;
}

dhs_status ht_set_phase_timing(dhs_table* t, int enable) {
  DHS_TRY(check_table(t));
  if (enable < 0 || enable > 2) return DHS_ERR_INVALID_ARG;
  t->timing = enable;
  return DHS_OK;
}

dhs_status ht_phase_times(dhs_table* t, double* ms_out, int64_t* count_out, int n) {
  DHS_TRY(check_table(t));
  if (n < 0 || (n > 0 && (!ms_out || !count_out))) return DHS_ERR_INVALID_ARG;
  DeviceGuard g(t->device);
  for (int i = 0; i < n; ++i) {
    ms_out[i] = 0.0;
    count_out[i] = 0;
  }
  dhs_status rc = DHS_OK;
  for (auto& r : t->recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) rc = DHS_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) rc = DHS_ERR_CUDA;
    if (r.phase < n) {
      ms_out[r.phase] += ms;
      count_out[r.phase] += 1;
    }
    t->ev_pool.push_back(r.a);
    t->ev_pool.push_back(r.b);
  }
  t->recs.clear();
  cudaGetLastError();
  return rc;
}


// ---------------------------------------------------------------------------
// Backward + update without any allocation
// ---------------------------------------------------------------------------
// For callers that cannot allocate device memory during a training step (for
// example a runtime that forbids cudaMalloc once its steps are running, or
// one that hands this library only the buffers it owns).  The scratch of the
// sort and the segment reduce lives in one file-scope device array of fixed
// size instead of the table's growable workspace.
}  // extern "C"

namespace {

constexpr long long kNoAllocMaxKeys = DHS_NOALLOC_MAX_KEYS;
constexpr int kNoAllocMaxDim = 128;
constexpr int kNoAllocMinChunk = 32;  // seg_chunk() never goes below this

constexpr size_t na_align(size_t x) { return (x + 255) & ~size_t(255); }
constexpr size_t kNaPairs = na_align(kNoAllocMaxKeys * 4);  // one of ka, va, kb, vb
constexpr size_t kNaSortZero = na_align(kSortZeroWords * 4);
constexpr size_t kNaStatus =
    na_align((size_t)kRadixMaxPasses * ((kNoAllocMaxKeys + kRadixTile - 1) / kRadixTile) * kRadixBins * 8);
constexpr size_t kNaChunks = (kNoAllocMaxKeys + kNoAllocMinChunk - 1) / kNoAllocMinChunk;
constexpr size_t kNaPart = na_align(kNaChunks * kNoAllocMaxDim * 8);  // one of part_head, part_tail
constexpr size_t kNaOwners = na_align(kNaChunks * 4);
constexpr size_t kNaPlan = na_align((6 * kNaChunks + combine_batch_cap(kNaChunks)) * 4);
constexpr size_t kNaSlots = na_align(combine_slot_cap(kNaChunks) * kNoAllocMaxDim * 8);
constexpr size_t kNoAllocScratchBytes =
    4 * kNaPairs + kNaSortZero + kNaStatus + 2 * kNaPart + kNaOwners + kNaPlan + kNaSlots;

// Every GPU that loads this library holds this array until the process exits.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[128] = {};

// Device address of the scratch array on `dev` (which must be current): looked
// up once per device with cudaGetSymbolAddress, then cached.
dhs_status noalloc_scratch(int dev, unsigned char** out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (dev < 0 || dev >= 128) return DHS_ERR_UNSUPPORTED;
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return DHS_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = (unsigned char*)g_noalloc_ptr[dev];
  return DHS_OK;
}

}  // namespace

extern "C" {

dhs_status embbag_backward_update_noalloc(dhs_table* t, const int64_t* d_keys, int64_t n_keys,
                                          const int64_t* d_bag_offsets, int64_t n_bags,
                                          const float* d_grad, float lr, dhs_stream stream) {
  DHS_TRY(check_table(t));
  if (n_keys < 0 || n_bags < 0 || n_bags >= (1ll << 31)) return DHS_ERR_INVALID_ARG;
  if (n_keys > kNoAllocMaxKeys || t->dim > kNoAllocMaxDim) return DHS_ERR_INVALID_ARG;
  // the partial vectors are sized for kNoAllocMaxDim doubles each
  if (seg_nv(t->dim) * seg_group(t->dim) * 4 > kNoAllocMaxDim) return DHS_ERR_INVALID_ARG;
  if (n_bags == 0 && n_keys != 0) return DHS_ERR_INVALID_ARG;
  if (n_bags > 0 && (!d_bag_offsets || !d_grad)) return DHS_ERR_INVALID_ARG;
  if ((uintptr_t)d_grad % 16) return DHS_ERR_INVALID_ARG;
  if (n_keys > 0 && !d_keys) return DHS_ERR_INVALID_ARG;
  if (!std::isfinite(lr)) return DHS_ERR_INVALID_ARG;
  DeviceGuard g(t->device);
  unsigned char* base = nullptr;
  DHS_TRY(noalloc_scratch(t->device, &base));
  cudaStream_t s = (cudaStream_t)stream;
  t->last_stream = s;
  t->adam_t += 1;
  t->bwd_n += n_keys;
  if (n_keys == 0) return DHS_OK;

  unsigned* ka = (unsigned*)base;
  unsigned* va = (unsigned*)(base + kNaPairs);
  unsigned* kb = (unsigned*)(base + 2 * kNaPairs);
  unsigned* vb = (unsigned*)(base + 3 * kNaPairs);
  unsigned* hist = (unsigned*)(base + 4 * kNaPairs);
  unsigned* tile_ctr = hist + kRadixMaxPasses * kRadixBins;
  unsigned long long* status = (unsigned long long*)(base + 4 * kNaPairs + kNaSortZero);
  double* part_head = (double*)(base + 4 * kNaPairs + kNaSortZero + kNaStatus);
  double* part_tail = (double*)(base + 4 * kNaPairs + kNaSortZero + kNaStatus + kNaPart);
  unsigned char* const tail = base + 4 * kNaPairs + kNaSortZero + kNaStatus + 2 * kNaPart;
  unsigned* owners = (unsigned*)tail;
  const CombinePlan plan =
      combine_plan((unsigned*)(tail + kNaOwners), (double*)(tail + kNaOwners + kNaPlan), kNaChunks, hist);

  refresh_ub(t, false);
  const unsigned sentinel = (unsigned)t->rows_ub;
  int bits = 0;
  while (bits < 32 && (1ull << bits) <= (unsigned long long)sentinel) ++bits;
  const int passes = std::min(kRadixMaxPasses, std::max(1, (bits + 7) / 8));

  {
    const int bpc = bwd_probe_bags(n_keys, n_bags);
    const long long warps = (n_bags + bpc - 1) / bpc;
    const long long grid = grid_for((warps + 7) / 8, resident_blocks(bwd_probe_kernel<false>, 256, 0, t->sm_count));
    const long long ntiles = (n_keys + kRadixTile - 1) / kRadixTile;
    // the shared array keeps the last call's counters: they start at zero
    DHS_CUDA(cudaMemsetAsync(hist, 0, (size_t)kSortZeroWords * 4, s));
    bwd_probe_kernel<false><<<(unsigned)grid, 256, 0, s>>>(idmap(t), (const long long*)d_keys, n_keys,
                                                    (const long long*)d_bag_offsets, n_bags, ka, va,
                                                    sentinel, hist, passes, status, ntiles * kRadixBins,
                                                    nullptr, 0, nullptr, 0, bpc, nullptr, false, nullptr, nullptr,
                                                    nullptr, nullptr, t->st);
    DHS_TRY(last_launch());
  }
  const long long ntiles = (n_keys + kRadixTile - 1) / kRadixTile;
  {
    for (int p = 0; p < passes; ++p) {
      const long long words = ntiles * kRadixBins;
      launch_k(radix_onesweep_kernel, (unsigned)ntiles, kRadixThreads, 0, s, 
          ka, va, kb, vb, n_keys, 8 * p, hist + p * kRadixBins, status + (long long)p * words, tile_ctr + p,
          status + (long long)(p + 1) * words, p + 1 < passes ? words : 0, t->st);
      DHS_TRY(last_launch());
      std::swap(ka, kb);
      std::swap(va, vb);
    }
  }
  OptArgs oa;
  oa.opt = t->opt;
  oa.lr = lr;
  oa.eps = t->eps;
  oa.b1 = t->b1;
  oa.b2 = t->b2;
  oa.c1 = (float)(1.0 - (double)t->b1);
  oa.c2 = (float)(1.0 - (double)t->b2);
  oa.bc1 = (float)(1.0 - std::pow((double)t->b1, (double)t->adam_t));
  oa.bc2 = (float)(1.0 - std::pow((double)t->b2, (double)t->adam_t));
  const int G = seg_group(t->dim), NV = seg_nv(t->dim);
  const int chunk = seg_chunk(n_keys);
  RunTable no_table{};  // the owner chunks go to the combine kernels as they close
  DHS_TRY(launch_seg(t, ka, va, n_keys, d_grad, n_bags, oa, part_head, part_tail, hist + kSegChunkCtrWord, owners,
                     hist + kSegOwnerCtrWord, nullptr, nullptr, false, no_table, s));
  t->n_launches += 1 + passes;
  return launch_combine(t, ka, n_keys, oa, part_head, part_tail, chunk, NV * G * 4, owners, hist, plan, s);
}

// ---- hash-sharded engine ----

dhs_status ht_shard_route(dhs_table* t, const int64_t* d_keys, int64_t n_keys, int32_t world,
                          int64_t* d_send_keys, int32_t* d_slot_of, int64_t* h_send_counts, dhs_stream stream) {
  DHS_TRY(check_table(t));
  if (world < 1 || world > kRadixBins || n_keys < 0 || n_keys >= (1ll << 31) || !h_send_counts)
    return DHS_ERR_INVALID_ARG;
  if (n_keys > 0 && (!d_keys || !d_send_keys || !d_slot_of)) return DHS_ERR_INVALID_ARG;
  for (int r = 0; r < world; ++r) h_send_counts[r] = 0;
  if (n_keys == 0) return DHS_OK;
  DeviceGuard g(t->device);
  cudaStream_t s = (cudaStream_t)stream;
  t->last_stream = s;
  DHS_TRY(ensure_ws(t, n_keys, s));
  // owner histogram (256 bins) and the routing pass's tile counter
  DHS_TRY(bget(t, t->b_shard, (size_t)(kRadixBins + 1) * 4, s));
  unsigned* hist = (unsigned*)t->b_shard.p;
  DHS_CUDA(cudaMemsetAsync(hist, 0, t->b_shard.bytes, s));
  unsigned* okey = (unsigned*)t->b_ka.p;
  unsigned* opos = (unsigned*)t->b_va.p;
  unsigned* skey = (unsigned*)t->b_kb.p;
  unsigned* spos = (unsigned*)t->b_vb.p;
  const long long ntiles = (n_keys + kRadixTile - 1) / kRadixTile;
  unsigned long long* status = (unsigned long long*)t->b_totals.p;
  const unsigned grid = (unsigned)std::min<long long>((n_keys + 255) / 256, (long long)t->sm_count * 8);
  // owners + positions, one stable digit pass by owner, then the gather
  (void)launch_k(shard_count_kernel, grid, 256, 0, s, (const long long*)d_keys, (long long)n_keys,
                 (unsigned)world, okey, opos, hist, status, ntiles * kRadixBins);
  DHS_TRY(last_launch());
  (void)launch_k(radix_onesweep_kernel, (unsigned)ntiles, kRadixThreads, 0, s, (const unsigned*)okey,
                 (const unsigned*)opos, skey, spos, (long long)n_keys, 0, (const unsigned*)hist, status,
                 hist + kRadixBins, (unsigned long long*)nullptr, 0ll, t->st);
  DHS_TRY(last_launch());
  (void)launch_k(shard_gather_kernel, grid, 256, 0, s, (const long long*)d_keys, (const unsigned*)spos,
                 (long long)n_keys, (long long*)d_send_keys, (int*)d_slot_of);
  DHS_TRY(last_launch());
  t->n_launches += 3;
  std::vector<unsigned> counts(world);
  DHS_CUDA(cudaMemcpyAsync(counts.data(), hist, world * sizeof(unsigned), cudaMemcpyDeviceToHost, s));
  DHS_CUDA(cudaStreamSynchronize(s));
  for (int r = 0; r < world; ++r) h_send_counts[r] = counts[r];
  return DHS_OK;
}

dhs_status ht_shard_pool(dhs_table* t, const float* d_rows, const int32_t* d_slot_of, int64_t n_keys,
                         const int64_t* d_bag_offsets, int64_t n_bags, const float* d_per_sample_weights,
                         dhs_pool_mode mode, float* d_pooled_out, dhs_stream stream) {
  DHS_TRY(check_table(t));
  if (n_keys < 0 || n_keys >= (1ll << 31) || n_bags < 0 || n_bags >= (1ll << 31)) return DHS_ERR_INVALID_ARG;
  if (mode != DHS_POOL_SUM && mode != DHS_POOL_MEAN) return DHS_ERR_INVALID_ARG;
  if (mode == DHS_POOL_MEAN && d_per_sample_weights) return DHS_ERR_INVALID_ARG;
  if (n_bags == 0) return n_keys == 0 ? DHS_OK : DHS_ERR_INVALID_ARG;
  if (!d_bag_offsets || !d_pooled_out || (n_keys > 0 && (!d_rows || !d_slot_of))) return DHS_ERR_INVALID_ARG;
  if ((uintptr_t)d_pooled_out % 16 || (uintptr_t)d_rows % 16) return DHS_ERR_INVALID_ARG;
  DeviceGuard g(t->device);
  cudaStream_t s = (cudaStream_t)stream;
  t->last_stream = s;
  const float* psw = n_keys > 0 ? d_per_sample_weights : nullptr;
  const unsigned grid = (unsigned)std::min<long long>((n_bags + 7) / 8, (long long)t->sm_count * 8);
  auto k = psw ? shard_pool_kernel<true, false>
               : (mode == DHS_POOL_MEAN ? shard_pool_kernel<false, true> : shard_pool_kernel<false, false>);
  (void)launch_k(k, grid, 256, 0, s, d_rows, (const int*)d_slot_of, (long long)n_keys,
                 (const long long*)d_bag_offsets, (long long)n_bags, t->dim, psw, d_pooled_out, t->st);
  t->n_launches++;
  return last_launch();
}

dhs_status ht_shard_grads(dhs_table* t, const float* d_grad, const int64_t* d_bag_offsets, int64_t n_bags,
                          int64_t n_keys, const int32_t* d_slot_of, const float* d_per_sample_weights,
                          dhs_pool_mode mode, float* d_send_grads, float* d_send_fact, dhs_stream stream) {
  DHS_TRY(check_table(t));
  if (n_keys < 0 || n_keys >= (1ll << 31) || n_bags < 0 || n_bags >= (1ll << 31)) return DHS_ERR_INVALID_ARG;
  if (mode != DHS_POOL_SUM && mode != DHS_POOL_MEAN) return DHS_ERR_INVALID_ARG;
  if (mode == DHS_POOL_MEAN && d_per_sample_weights) return DHS_ERR_INVALID_ARG;
  if (n_bags == 0) return n_keys == 0 ? DHS_OK : DHS_ERR_INVALID_ARG;
  if (!d_bag_offsets || !d_grad || (n_keys > 0 && (!d_slot_of || !d_send_grads))) return DHS_ERR_INVALID_ARG;
  if ((uintptr_t)d_grad % 16 || (uintptr_t)d_send_grads % 16) return DHS_ERR_INVALID_ARG;
  const float* psw = n_keys > 0 ? d_per_sample_weights : nullptr;
  const int fact = psw ? 1 : (mode == DHS_POOL_MEAN ? 2 : 0);
  if (fact && n_keys > 0 && !d_send_fact) return DHS_ERR_INVALID_ARG;
  DeviceGuard g(t->device);
  cudaStream_t s = (cudaStream_t)stream;
  t->last_stream = s;
  const unsigned grid = (unsigned)std::min<long long>((n_bags + 7) / 8, (long long)t->sm_count * 8);
  auto k = fact == 1 ? shard_expand_kernel<1> : (fact == 2 ? shard_expand_kernel<2> : shard_expand_kernel<0>);
  (void)launch_k(k, grid, 256, 0, s, d_grad, (const long long*)d_bag_offsets, (long long)n_bags, (long long)n_keys,
                 (const int*)d_slot_of, psw, t->dim, d_send_grads, d_send_fact, t->st);
  t->n_launches++;
  return last_launch();
}

}  // extern "C"
