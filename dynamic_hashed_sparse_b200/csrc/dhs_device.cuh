// Device-side definitions of the dynamic hashed embedding engine (sm_100a).
//
// IDMap ([RecIS] overview, "Embedding Engine": first-level store from feature
// id to memory offset): open addressing over 16-byte slots {key, val}, probed
// in 32-byte windows (two slots = one DRAM sector), windows visited linearly.
// An empty slot is all ones (key -1, val all ones).  During a forward call a
// key claimed in that call holds val = PENDING | (smallest batch position
// that carries it); the offset assignment that follows replaces it with the
// row offset.
//
// EmbeddingBlocks ([RecIS] overview, second level: contiguous blocks holding
// parameters and optimizer state, appended as the table grows): a device
// array of block pointers; row r lives at blocks[r >> log2_block_rows] +
// (r & (block_rows - 1)) * stride, stride = the weights (wfl floats: dim
// fp32 values, or dim bf16 values in dim / 2 floats) + the optimizer state
// (fp32), a multiple of 4 floats so every row is 16-byte aligned.
#pragma once

#include <climits>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

//   DHS_PDL 1: the hot-path kernels are launched as programmatic dependents of
//           the kernel before them in the stream (their launch overlaps its
//           tail); 0: plain launches
#ifndef DHS_PDL
#define DHS_PDL 1
#endif

namespace dhs {

// First statement of a hot-path kernel.  Launched as a programmatic
// dependent, the kernel waits here until the kernel before it in the stream
// has finished and its writes are visible (a no-op after a plain launch);
// then it lets the kernel after it begin launching, whose blocks in turn wait
// at their own first statement.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

constexpr unsigned long long kEmptyKey = ~0ull;
// An evicted key's slot: probes step over it (the chain goes on), and it is
// never claimed again (so no key can sit behind an empty slot in its chain);
// a rehash drops it.
constexpr unsigned long long kTombKey = ~1ull;
constexpr unsigned long long kPending = 1ull << 63;
// Between calls, the value of a key that is known but has no row yet (not
// admitted): above every PENDING | position, so a claim's atomicMin replaces it.
constexpr unsigned long long kCounting = ~1ull;
// The forward's per-position record of a key without a row (known but not
// admitted, or not placed because the table was full).
constexpr long long kRecNoRow = LLONG_MIN;

struct __align__(16) Slot {
  unsigned long long key;
  unsigned long long val;
};

// Device-resident scalars of one table.
struct DevState {
  unsigned long long row_count;  // rows assigned so far
  unsigned long long keys_used;  // slots claimed since the last rehash (with admission / eviction)
  unsigned long long row_base;   // first appended row of the current call's new keys
  unsigned long long m_last;     // new rows of the last insert call
  unsigned long long n_blocks;   // blocks the host has appended
  unsigned long long sum_new;    // total inserted rows
  unsigned long long sum_unique; // total distinct keys updated by backward calls
  unsigned long long free_count; // rows in the free list (evicted rows)
  unsigned long long free_head;  // free-list rows handed out so far
  unsigned long long free_base;  // free_head before the current call
  unsigned long long m_free;     // rows of the current call taken from the free list
  unsigned int err;              // first latched error code, 0 = none
  unsigned int ticket;           // last-block-done counter (mark kernel)
  unsigned int ticket2;          // last-block-done counter (free-list compaction)
  unsigned int pad;
  unsigned int fwd_ctr[2];       // chunk counters of the forward's pool kernels (one per call, alternating)
};

enum : unsigned { kErrInvalid = 1u, kErrFull = 4u, kErrNotFound = 5u, kErrInternal = 7u };

__device__ __forceinline__ void latch(DevState* st, unsigned code) {
  if (*(volatile unsigned*)&st->err == 0u) atomicCAS(&st->err, 0u, code);
}

// Bucket hash: the 64-bit finaliser of MurmurHash3 (A. Appleby, public
// domain).  Only the probe start depends on it, never a result.
__device__ __forceinline__ unsigned long long hash_key(unsigned long long k) {
  k ^= k >> 33;
  k *= 0xff51afd7ed558ccdull;
  k ^= k >> 33;
  k *= 0xc4ceb9fe1a85ec53ull;
  k ^= k >> 33;
  return k;
}

// Output number n (n >= 1) of the splitmix64 generator seeded with `seed`
// (Steele, Lea & Flood, OOPSLA 2014; Vigna's splitmix64.c): the state after n
// steps is seed + n * golden gamma (mod 2^64), passed through the mixer.
constexpr unsigned long long kSplitmixGamma = 0x9E3779B97F4A7C15ull;
constexpr unsigned long long kSplitmixM1 = 0xBF58476D1CE4E5B9ull;
constexpr unsigned long long kSplitmixM2 = 0x94D049BB133111EBull;

// Bits 40..63 of splitmix64's output for the generator state z (the state
// after its gamma step).  The finaliser's last step, x ^ (x >> 31), leaves
// bits 40..63 of x unchanged, so they are the top 24 bits of the second
// product, of which only the high word is formed:
// hi32(lo64(a * m)) = hi32(alo * mlo) + alo * mhi + ahi * mlo (mod 2^32).
__device__ __forceinline__ unsigned splitmix64_top24(unsigned long long z) {
  z = (z ^ (z >> 30)) * kSplitmixM1;
  z ^= z >> 27;
  const unsigned lo = (unsigned)z, hi = (unsigned)(z >> 32);
  const unsigned top = __umulhi(lo, (unsigned)kSplitmixM2) + lo * (unsigned)(kSplitmixM2 >> 32) +
                       hi * (unsigned)kSplitmixM2;
  return top >> 8;
}

// Initial weight from 24 random bits: centred, times 0.05 * 2^-23 (one
// rounded fp32 multiply of exact operands), a value in [-0.05, 0.05).
__device__ __forceinline__ float init_from_top24(unsigned t) {
  return __fmul_rn((float)((int)t - (1 << 23)), 0.05f * 0x1p-23f);
}

// Initial weights j .. j+3 of the row of `key`: weight j comes from the
// (j+1)-th splitmix64 output seeded with the key, whose state is
// key + (j+1) * gamma.
__device__ __forceinline__ float4 init_weight4(unsigned long long key, int j) {
  const unsigned long long z = key + (unsigned long long)(j + 1) * kSplitmixGamma;
  return make_float4(init_from_top24(splitmix64_top24(z)),
                     init_from_top24(splitmix64_top24(z + kSplitmixGamma)),
                     init_from_top24(splitmix64_top24(z + 2 * kSplitmixGamma)),
                     init_from_top24(splitmix64_top24(z + 3 * kSplitmixGamma)));
}

struct IdMap {
  Slot* slots;
  unsigned long long win_mask;  // windows - 1 (windows = slots / 2, a power of two)
};

struct RowSpace {
  float* const* blocks;
  unsigned long long br_mask;  // block_rows - 1
  int log2_br;
  int stride;  // floats per row
  int wfl;     // floats holding the weights (dim, or dim / 2 for bf16 weights); the state starts there
  __device__ __forceinline__ float* row(unsigned long long r) const {
    float* b = (float*)__ldg((const unsigned long long*)(blocks + (r >> log2_br)));
    return b + (r & br_mask) * (unsigned long long)stride;
  }
};

// Arrivals of the pieces of the long segments of one backward: open
// addressing on the row (mask + 1 entries, a power of two).  key = row + 1
// (0: empty), ctr = the pieces' arrival sum, c0 / c1 = the segment's first and
// last sort chunk.  key and ctr start at zero.  key == nullptr: no table (the
// owner chunks go to the combine kernels as they close).
struct RunTable {
  unsigned* key;
  unsigned* ctr;
  unsigned* c0;
  unsigned* c1;
  unsigned mask;
  unsigned max_pieces;  // longer segments are finished by the combine kernels
};

enum : int { kHit = 0, kNew = 1, kBad = 2 };

// Admission / eviction state of a table (null pointers and zeros when the
// table uses neither).
struct Hooks {
  unsigned* cnt;              // [slots] occurrences of keys without a row (admission)
  unsigned* stamp;            // [slots] last insert call a key occurred in (eviction)
  unsigned admit;             // admission threshold (<= 1: a row at first sight)
  unsigned step;              // this insert call's number (1, 2, ...)
  const unsigned* free_list;  // rows freed by evictions, ascending
  unsigned* free_bm;          // bit per row: the row is free
};

// Find `key`, claiming an empty slot if it is absent.  Returns kHit with the
// row offset in `out`, or kNew with the slot index in `out` (the key has no
// row yet: new in this call, or known but not admitted; the slot's val
// becomes PENDING | min position).  `slot` receives the key's slot index.
// No thread ever waits on another: a claimed key is usable at once, its
// offset is assigned by a later kernel.  The probe visits at most every
// window once; tombstones are stepped over and never claimed.  `claimed`
// is set when this thread took an empty slot.
__device__ __forceinline__ int probe_claim(IdMap m, unsigned long long key, unsigned pos,
                                           unsigned long long& out, unsigned long long& slot,
                                           bool& claimed, DevState* st) {
  unsigned long long w = hash_key(key) & m.win_mask;
  const unsigned long long mine = kPending | (unsigned long long)pos;
  claimed = false;
  for (unsigned long long step = 0; step <= m.win_mask; ++step) {
    Slot* ws = m.slots + 2 * w;
    const ulonglong2 a = *reinterpret_cast<const ulonglong2*>(ws);
    const ulonglong2 b = *reinterpret_cast<const ulonglong2*>(ws + 1);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const unsigned long long k = j ? b.x : a.x;
      const unsigned long long v = j ? b.y : a.y;
      if (k == key) {
        slot = 2 * w + j;
        if (!(v & kPending)) {
          out = v;
          return kHit;
        }
        if (mine < v) atomicMin(&ws[j].val, mine);
        out = slot;
        return kNew;
      }
      if (k == kEmptyKey) {
        const unsigned long long old = atomicCAS(&ws[j].key, kEmptyKey, key);
        if (old == kEmptyKey || old == key) {
          atomicMin(&ws[j].val, mine);
          slot = 2 * w + j;
          out = slot;
          claimed = old == kEmptyKey;
          return kNew;
        }
      }
    }
    w = (w + 1) & m.win_mask;
  }
  latch(st, kErrFull);
  return kBad;
}

__device__ __forceinline__ int probe_claim(IdMap m, unsigned long long key, unsigned pos,
                                           unsigned long long& out, DevState* st) {
  unsigned long long slot;
  bool claimed;
  return probe_claim(m, key, pos, out, slot, claimed, st);
}

// Read-only probe (no concurrent writers): the row offset; -1 if the key is
// absent; -2 if it is known but has no row (not admitted yet, or left
// without a row by a failed assignment).  Tombstones are stepped over.
__device__ __forceinline__ long long probe_find(IdMap m, unsigned long long key) {
  unsigned long long w = hash_key(key) & m.win_mask;
  for (unsigned long long step = 0; step <= m.win_mask; ++step) {
    const ulonglong2* ws = reinterpret_cast<const ulonglong2*>(m.slots + 2 * w);
    const ulonglong2 a = __ldg(ws);
    const ulonglong2 b = __ldg(ws + 1);
    if (a.x == key) return (a.y & kPending) ? -2 : (long long)a.y;
    if (a.x == kEmptyKey) return -1;
    if (b.x == key) return (b.y & kPending) ? -2 : (long long)b.y;
    if (b.x == kEmptyKey) return -1;
    w = (w + 1) & m.win_mask;
  }
  return -1;
}

// Bulk prefetch of `bytes` (a multiple of 16, 16-byte aligned) into L2: one
// instruction per row, no register or shared-memory cost, so a warp can put a
// whole window of upcoming rows in flight.
__device__ __forceinline__ void prefetch_l2(const void* p, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// bf16 weights.  A bf16 value is the top half of an fp32, so widening is
// exact; storing rounds to nearest, ties to even.
__device__ __forceinline__ float bf16_lo(unsigned w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(unsigned w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float round_bf16(float a) { return __bfloat162float(__float2bfloat16_rn(a)); }
// two values rounded to bf16, a in the low half
__device__ __forceinline__ unsigned pack_bf16x2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const unsigned*>(&v);
}
// 8 bf16 weights (one 16-byte unit) widened to fp32
__device__ __forceinline__ void unpack_bf16x8(const uint4 u, float4& a, float4& b) {
  a = make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
  b = make_float4(bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w));
}

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
  return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z),
                     __fadd_rn(a.w, b.w));
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ unsigned warp_sum_u32(unsigned v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace dhs
