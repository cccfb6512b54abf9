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
// (r & (block_rows - 1)) * stride, stride = dim weights + optimizer state,
// a multiple of 4 floats so every row is 16-byte aligned.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace dhs {

constexpr unsigned long long kEmptyKey = ~0ull;
constexpr unsigned long long kPending = 1ull << 63;

struct __align__(16) Slot {
  unsigned long long key;
  unsigned long long val;
};

// Device-resident scalars of one table.
struct DevState {
  unsigned long long row_count;  // rows assigned so far
  unsigned long long row_base;   // first row of the current call's new keys
  unsigned long long m_last;     // new rows of the last insert call
  unsigned long long n_blocks;   // blocks the host has appended
  unsigned long long sum_new;    // total inserted rows
  unsigned long long sum_unique; // total distinct keys updated by backward calls
  unsigned int err;              // first latched error code, 0 = none
  unsigned int ticket;           // last-block-done counter (mark kernel)
  unsigned int ticket2;          // spare
  unsigned int pad;
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
  __device__ __forceinline__ float* row(unsigned long long r) const {
    float* b = (float*)__ldg((const unsigned long long*)(blocks + (r >> log2_br)));
    return b + (r & br_mask) * (unsigned long long)stride;
  }
};

enum : int { kHit = 0, kNew = 1, kBad = 2 };

// Find `key`, claiming an empty slot if it is absent.  Returns kHit with the
// row offset in `out`, or kNew with the slot index in `out` (the key is new in
// this call; the slot's val becomes PENDING | min position).  No thread ever
// waits on another: a claimed key is usable at once, its offset is assigned
// by a later kernel.  The probe visits at most every window once.
__device__ __forceinline__ int probe_claim(IdMap m, unsigned long long key, unsigned pos,
                                           unsigned long long& out, DevState* st) {
  unsigned long long w = hash_key(key) & m.win_mask;
  const unsigned long long mine = kPending | (unsigned long long)pos;
  for (unsigned long long step = 0; step <= m.win_mask; ++step) {
    Slot* ws = m.slots + 2 * w;
    const ulonglong2 a = *reinterpret_cast<const ulonglong2*>(ws);
    const ulonglong2 b = *reinterpret_cast<const ulonglong2*>(ws + 1);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const unsigned long long k = j ? b.x : a.x;
      const unsigned long long v = j ? b.y : a.y;
      if (k == key) {
        if (!(v & kPending)) {
          out = v;
          return kHit;
        }
        if (mine < v) atomicMin(&ws[j].val, mine);
        out = 2 * w + j;
        return kNew;
      }
      if (k == kEmptyKey) {
        const unsigned long long old = atomicCAS(&ws[j].key, kEmptyKey, key);
        if (old == kEmptyKey || old == key) {
          atomicMin(&ws[j].val, mine);
          out = 2 * w + j;
          return kNew;
        }
      }
    }
    w = (w + 1) & m.win_mask;
  }
  latch(st, kErrFull);
  return kBad;
}

// Read-only probe (no concurrent writers): row offset, or -1 if absent (or
// left without a row by a failed assignment).
__device__ __forceinline__ long long probe_find(IdMap m, unsigned long long key) {
  unsigned long long w = hash_key(key) & m.win_mask;
  for (unsigned long long step = 0; step <= m.win_mask; ++step) {
    const ulonglong2* ws = reinterpret_cast<const ulonglong2*>(m.slots + 2 * w);
    const ulonglong2 a = __ldg(ws);
    const ulonglong2 b = __ldg(ws + 1);
    if (a.x == key) return (a.y & kPending) ? -1 : (long long)a.y;
    if (a.x == kEmptyKey) return -1;
    if (b.x == key) return (b.y & kPending) ? -1 : (long long)b.y;
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
