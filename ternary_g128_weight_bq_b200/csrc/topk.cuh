// topk.cuh -- selection of the k largest logits inside the GEMV kernels (k <= 32), and the draw of
// a token from them.
//
// Model card "prism-ml/Bonsai-27B-mlx-1bit", section "Generation parameters": top-k 20, top-p
// 0.95, temperature 0.7. A logit is carried as a 64-bit key that orders like (value descending,
// index ascending): the float's bits made monotone (negatives inverted, positives with the sign
// bit set) in the high half and 0xFFFFFFFF - index in the low half. Keys are unique, so "the k
// largest keys" is one well-defined set.
//
// Selection is a radix select over the keys, 8 bits at a time from the top, by all threads of
// a named barrier: each pass builds a 256-bin histogram (shared-memory atomics) of the next 8
// bits of the keys that share the prefix chosen so far; one warp finds the bin where the count
// from the top reaches the number of keys still missing and extends the prefix with it. Once the
// keys at or above the bottom of that bin are at most 64 (usually after one or two passes for
// logits), they are gathered and ranked, one thread per key counting the larger ones.
#pragma once

#include <stdint.h>

namespace bq {
namespace topk {

constexpr int kMaxK = 32;
constexpr int kGather = 64;

struct Smem {
    uint32_t hist[256];
    unsigned long long buf[kGather];
    unsigned long long prefix;    // chosen bits so far (top plen bits), low bits zero
    int plen;                     // number of chosen bits
    int need;                     // keys still to select among those matching the prefix
    int gather;                   // 1: gather keys >= prefix now
    int cnt;                      // gathered keys
    int last;                     // this CTA drew the last ticket
    unsigned long long floor[8];  // the merge's floor per token row: the largest of the CTAs' k-th keys
};

__device__ __forceinline__ unsigned long long key_of(float v, uint32_t index)
{
    const uint32_t u = __float_as_uint(v);
    const uint32_t m = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)m << 32) | (0xFFFFFFFFu - index);
}

__device__ __forceinline__ float value_of(unsigned long long key)
{
    const uint32_t m = (uint32_t)(key >> 32);
    return __uint_as_float((m & 0x80000000u) ? (m & 0x7FFFFFFFu) : ~m);
}

__device__ __forceinline__ uint32_t index_of(unsigned long long key) { return 0xFFFFFFFFu - (uint32_t)key; }

template <int NT>
__device__ __forceinline__ void bar(int id)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(NT) : "memory");
}

// The k largest of the n keys key_at(0 .. n-1) (n >= k), descending, into out[0 .. k) (shared
// memory). NT threads (tid in [0, NT), a multiple of 32) take part; they synchronise on named
// barrier `id`.
template <int NT, class KeyAt>
__device__ void select(KeyAt key_at, int n, int k, Smem *sm, unsigned long long *out, int tid, int id)
{
    const int lane = tid & 31;
    if (tid == 0) {
        sm->prefix = 0ull;
        sm->plen = 0;
        sm->need = k;
        sm->gather = 0;
        sm->cnt = 0;
    }
    bar<NT>(id);
    while (true) {
        const int plen = sm->plen;
        const unsigned long long prefix = sm->prefix;
        for (int b = tid; b < 256; b += NT)
            sm->hist[b] = 0u;
        bar<NT>(id);
        const int shift = 56 - plen;
        // logits crowd into a few bins: the lanes of a warp that hit the same bin add once
        for (int i0 = tid - lane; i0 < n; i0 += NT) {
            const int i = i0 + lane;
            int bin = -1;
            if (i < n) {
                const unsigned long long key = key_at(i);
                if (plen == 0 || (key >> (64 - plen)) == (prefix >> (64 - plen)))
                    bin = (int)((key >> shift) & 255u);
            }
            const unsigned same = __match_any_sync(0xffffffffu, bin);
            if (bin >= 0 && lane == __ffs(same) - 1)
                atomicAdd(&sm->hist[bin], (uint32_t)__popc(same));
        }
        bar<NT>(id);
        if (tid < 32) {
            // lane l holds bins 255 - 8 l .. 248 - 8 l (descending)
            uint32_t h[8], s = 0;
#pragma unroll
            for (int j = 0; j < 8; j++) {
                h[j] = sm->hist[255 - 8 * lane - j];
                s += h[j];
            }
            uint32_t incl = s;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t o = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d)
                    incl += o;
            }
            const uint32_t excl = incl - s;
            const uint32_t need = (uint32_t)sm->need;
            const bool mine = excl < need && need <= incl;
            if (mine) {
                // the bin (of this lane's 8, descending) where the running count reaches need;
                // unrolled, so h stays in registers
                uint32_t above = excl, hsel = 0;
                int jsel = 0;
                bool found = false;
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    if (!found) {
                        if (above + h[j] >= need) {
                            found = true;
                            jsel = j;
                            hsel = h[j];
                        } else {
                            above += h[j];
                        }
                    }
                }
                const uint32_t bin = 255u - 8u * lane - (uint32_t)jsel;
                const int need2 = (int)(need - above);
                const unsigned long long p2 = prefix | ((unsigned long long)bin << shift);
                sm->prefix = p2;
                sm->plen = plen + 8;
                sm->need = need2;
                // keys at or above the bottom of this bin: the k - need2 already above, plus its own
                sm->gather = (k - need2) + (int)hsel <= kGather || plen + 8 == 64;
            }
        }
        bar<NT>(id);
        if (sm->gather)
            break;
    }
    // gather every key >= prefix (prefix has zeros below the chosen bits)
    const unsigned long long lo = sm->prefix;
    for (int i = tid; i < n; i += NT) {
        const unsigned long long key = key_at(i);
        if (key >= lo) {
            const int slot = atomicAdd(&sm->cnt, 1);
            if (slot < kGather)
                sm->buf[slot] = key;
        }
    }
    bar<NT>(id);
    // rank of each gathered key = the number of larger ones (keys are unique); one thread per key,
    // every thread reading the same entry at a time (a shared-memory broadcast)
    const int cnt = sm->cnt < kGather ? sm->cnt : kGather;
    if (tid < cnt) {
        const unsigned long long a = sm->buf[tid];
        int r = 0;
        for (int j = 0; j < cnt; j++)
            r += sm->buf[j] > a;
        if (r < k)
            out[r] = a;
    }
    bar<NT>(id);
}

// Token drawn from k <= 32 candidates (keys descending, in shared memory) by one warp:
// probabilities softmax(v / T) over the k, the shortest leading run reaching top_p kept, then the
// first kept candidate whose renormalised cumulative probability exceeds u.
__device__ __forceinline__ int draw(const unsigned long long *keys, int k, float T, float top_p, float u, int lane)
{
    const float v0 = value_of(keys[0]);
    const float v = lane < k ? value_of(keys[lane]) : v0;
    float p = lane < k ? __expf((v - v0) / T) : 0.f;
    float c = p;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, c, d);
        if (lane >= d)
            c += o;
    }
    const float z = __shfl_sync(0xffffffffu, c, 31);
    // kept: lanes up to and including the first whose cumulative share reaches top_p
    const unsigned reach = __ballot_sync(0xffffffffu, lane < k && c >= top_p * z);
    const int keep = reach ? __ffs(reach) : k;
    const float kept = __shfl_sync(0xffffffffu, c, keep - 1);
    const unsigned over = __ballot_sync(0xffffffffu, lane < keep && c > u * kept);
    const int pick = over ? __ffs(over) - 1 : keep - 1;
    return (int)index_of(keys[pick]);
}

}  // namespace topk
}  // namespace bq
