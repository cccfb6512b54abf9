// Kernels of the hash-sharded engine ([RecIS] code-architecture section:
// collective All-to-All for parameter aggregation; [DLRM-E] practice cases 1
// and 2: embedding rows split across cards, lookups exchanged all-to-all).
// A rank routes its batch's ids to the keys' owners, pools the rows they send
// back, and sends each id's gradient row to its owner; the owners run the
// table's own forward and backward on what they receive.  The exchange itself
// is the caller's (NCCL all-to-all).
#pragma once

#include "dhs_device.cuh"
#include "dhs_fwd.cuh"

namespace dhs {

// Owner of key k among `world` ranks: the upper 32 bits of the splitmix64
// finaliser of k XOR a salt, scaled to [0, world) by a multiply-high.  The
// IDMap's bucket hash is a different function (MurmurHash3's finaliser), so
// the keys of one shard still spread over all of its buckets.
constexpr unsigned long long kShardSalt = 0x5DEECE66Dull;

__device__ __forceinline__ unsigned shard_owner(unsigned long long key, unsigned world) {
  unsigned long long z = key ^ kShardSalt;
  z = (z ^ (z >> 30)) * kSplitmixM1;
  z = (z ^ (z >> 27)) * kSplitmixM2;
  z ^= z >> 31;
  return (unsigned)(((z >> 32) * (unsigned long long)world) >> 32);
}

// Every position's owner (the routing pass's sort key, a negative key goes to
// rank 0 whose table call then reports it) and the position itself (its
// value); the owners' histogram (hist: 256 bins, zero on entry); the routing
// pass's look-back words cleared.
__global__ void __launch_bounds__(256)
shard_count_kernel(const long long* __restrict__ keys, long long n, unsigned world, unsigned* __restrict__ okey,
                   unsigned* __restrict__ opos, unsigned* __restrict__ hist,
                   unsigned long long* __restrict__ status, long long status_words) {
  pdl_enter();
  __shared__ unsigned h[256];
  h[threadIdx.x] = 0u;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < status_words;
       i += (long long)gridDim.x * blockDim.x)
    status[i] = 0ull;
  __syncthreads();
  for (long long p = (long long)blockIdx.x * blockDim.x + threadIdx.x; p < n; p += (long long)gridDim.x * blockDim.x) {
    const long long k = __ldg(keys + p);
    const unsigned o = k >= 0 ? shard_owner((unsigned long long)k, world) : 0u;
    okey[p] = o;
    opos[p] = (unsigned)p;
    atomicAdd(&h[o], 1u);
  }
  __syncthreads();
  const unsigned v = h[threadIdx.x];
  if (v) atomicAdd(hist + threadIdx.x, v);
}

// Keys in routed order and each position's slot in it (spos: positions
// sorted stably by owner).
__global__ void __launch_bounds__(256)
shard_gather_kernel(const long long* __restrict__ keys, const unsigned* __restrict__ spos, long long n,
                    long long* __restrict__ send_keys, int* __restrict__ slot_of) {
  pdl_enter();
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const unsigned p = __ldg(spos + i);
    send_keys[i] = __ldg(keys + p);
    slot_of[p] = (int)i;
  }
}

// Bag b's id range [s, e), clamped into [0, n]; malformed offsets latch
// kErrInvalid (as the table's own kernels do).
__device__ __forceinline__ void shard_bag(const long long* __restrict__ bo, long long b, long long nb, long long n,
                                          long long& s, long long& e, DevState* st) {
  s = __ldg(bo + b);
  e = __ldg(bo + b + 1);
  if (s < 0 || e < s || e > n || (b == 0 && s != 0) || (b + 1 == nb && e != n)) latch(st, kErrInvalid);
  s = min(max(s, 0ll), n);
  e = min(max(e, s), n);
}

// pooled[b] from the owners' rows, a warp per bag, each lane a float4
// column at a time: the ids of the bag in order, each row optionally
// multiplied by its weight (W), added in fp32; mean pooling divides once at
// the end -- the arithmetic of the table's own pooling kernels.
template <bool W, bool MEAN>
__global__ void __launch_bounds__(256)
shard_pool_kernel(const float* __restrict__ rows, const int* __restrict__ slot_of, long long n,
                  const long long* __restrict__ bo, long long nb, int dim, const float* __restrict__ psw,
                  float* __restrict__ out, DevState* st) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int d4 = dim >> 2;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long b = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; b < nb; b += nw) {
    long long s, e;
    shard_bag(bo, b, nb, n, s, e, st);
    for (int c = lane; c < d4; c += 32) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (long long p = s; p < e; ++p) {
        const int slot = __ldg(slot_of + p);
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (slot >= 0 && slot < n) x = __ldg(reinterpret_cast<const float4*>(rows + (long long)slot * dim) + c);
        else latch(st, kErrInvalid);
        if (W) {
          const float w = __ldg(psw + p);
          x = make_float4(__fmul_rn(w, x.x), __fmul_rn(w, x.y), __fmul_rn(w, x.z), __fmul_rn(w, x.w));
        }
        acc = f4add(acc, x);
      }
      __stcs(reinterpret_cast<float4*>(out + b * dim) + c, bag_out<MEAN>(acc, (int)(e - s)));
    }
  }
}

// Each id's gradient row (its bag's row of grad, copied) into its slot, and
// its factor: FACT 1 its weight, 2 its bag's length, 0 none.
template <int FACT>
__global__ void __launch_bounds__(256)
shard_expand_kernel(const float* __restrict__ grad, const long long* __restrict__ bo, long long nb, long long n,
                    const int* __restrict__ slot_of, const float* __restrict__ psw, int dim,
                    float* __restrict__ send_grads, float* __restrict__ send_fact, DevState* st) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int d4 = dim >> 2;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long b = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; b < nb; b += nw) {
    long long s, e;
    shard_bag(bo, b, nb, n, s, e, st);
    const float4* g = reinterpret_cast<const float4*>(grad + b * dim);
    for (long long p = s; p < e; ++p) {
      const int slot = __ldg(slot_of + p);
      if (slot < 0 || slot >= n) {
        if (lane == 0) latch(st, kErrInvalid);
        continue;
      }
      float4* o = reinterpret_cast<float4*>(send_grads + (long long)slot * dim);
      for (int c = lane; c < d4; c += 32) o[c] = __ldg(g + c);
      if (FACT != 0 && lane == 0) send_fact[slot] = FACT == 1 ? __ldg(psw + p) : (float)(e - s);
    }
  }
}

}  // namespace dhs
