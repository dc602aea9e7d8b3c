// Temperature / top-k sampling of the next token on the GPU, the variant beside the greedy
// argmax of both kernels' heads.
//
// A step's token is a function of (logits, temperature, top_k, seed, position) alone:
//   candidates  the top_k largest logits, in order of value (descending), then index (ascending)
//   weights     w_k = exp((z_k - z_0) / temperature)
//   draw        u = (splitmix64 output pos + 1 of the generator started from `seed`) >> 40, / 2^24
//   token       the first candidate whose cumulative weight exceeds u * (total weight)
// splitmix64 advances its state by 0x9E3779B97F4A7C15 and passes it through two
// xor-shift-multiply rounds and a final xor-shift (its published definition); output n of the
// generator started from state s is therefore mix(s + n * increment).
//
// The top-k selection is a radix select on order-preserving 32-bit keys of the values (8 bits
// per pass from the top: a 256-bin histogram of the keys that share the digits found so far),
// which gives the k-th largest key exactly; the winners are the keys above it plus, of the keys
// equal to it, those at the lowest positions. Callers lay out their values so that, among equal
// values, a lower position means a lower token index.
#pragma once
#include <math_constants.h>

#include "kie_device.cuh"

struct SampleScratch {
    unsigned hist[256];
    float win_v[KIE_TOPK_MAX];
    int win_p[KIE_TOPK_MAX];
    int win_i[KIE_TOPK_MAX];
    float top_v[KIE_TOPK_MAX];   // the winners in candidate order
    int top_i[KIE_TOPK_MAX];
    unsigned prefix, rem, gt;
    unsigned warp_sum[32];
};

// order-preserving key of a value; NaN below every number
KIE_DEV unsigned sample_key(float v) {
    const unsigned u = __float_as_uint(v);
    if (v != v) return 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

KIE_DEV unsigned long long splitmix64_output(unsigned long long seed, unsigned long long n) {
    unsigned long long z = seed + n * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// the draw of the step at position pos: a multiple of 2^-24 in [0, 1), exact in fp32
KIE_DEV float sample_uniform(unsigned long long seed, int pos) {
    return (float)(unsigned)(splitmix64_output(seed, (unsigned long long)pos + 1ull) >> 40) * (1.0f / 16777216.0f);
}

// Exclusive prefix sum of one count per thread over NT threads (NT a multiple of 32); the
// total lands in *total. Uses S.warp_sum and named barrier 1.
template <int NT>
KIE_DEV unsigned block_excl_scan(SampleScratch &S, unsigned c, unsigned *total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    unsigned incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) S.warp_sum[w] = incl;
    named_bar_sync(1, NT);
    unsigned base = 0, tot = 0;
    for (int k = 0; k < NT / 32; k++) {
        const unsigned v = S.warp_sum[k];
        if (k < w) base += v;
        tot += v;
    }
    *total = tot;
    named_bar_sync(1, NT);
    return base + incl - c;
}

// The k (1 <= k <= KIE_TOPK_MAX, k <= n) largest of n values, val(p) for position p, into
// S.top_v / S.top_i in candidate order, idx(p) giving a position's token index. All NT threads
// (0 .. NT-1, named barrier 1) call this with the same arguments.
template <int NT, class ValF, class IdxF>
__device__ __noinline__ void block_topk(SampleScratch &S, int n, int k, ValF val, IdxF idx) {
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid == 0) {
        S.prefix = 0u;
        S.rem = (unsigned)k;
        S.gt = 0u;
    }
    unsigned mask = 0u;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = tid; b < 256; b += NT) S.hist[b] = 0u;
        named_bar_sync(1, NT);
        const unsigned prefix = S.prefix;
        for (int p = tid; p < n; p += NT) {
            const unsigned key = sample_key(val(p));
            if ((key & mask) == prefix) atomicAdd(&S.hist[(key >> shift) & 255u], 1u);
        }
        named_bar_sync(1, NT);
        if (tid < 32) {
            // lane l holds digits 255 - 8l .. 248 - 8l, highest first; find the digit where the
            // count of keys at or above it first reaches the number still wanted
            const unsigned rem = S.rem;  // read before the shuffles (one lane writes it after them)
            unsigned c[8], s = 0;
#pragma unroll
            for (int j = 0; j < 8; j++) {
                c[j] = S.hist[255 - 8 * lane - j];
                s += c[j];
            }
            unsigned incl = s;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const unsigned before = incl - s;  // keys with a higher digit than this lane's
            const bool here = before < rem && incl >= rem;
            if (here) {
                unsigned acc = before;
                for (int j = 0; j < 8; j++) {
                    if (acc + c[j] >= rem) {
                        S.prefix = prefix | ((unsigned)(255 - 8 * lane - j) << shift);
                        S.rem = rem - acc;
                        break;
                    }
                    acc += c[j];
                }
            }
        }
        mask |= 255u << shift;
        named_bar_sync(1, NT);
    }
    const unsigned kth = S.prefix, need = S.rem;  // need >= 1 keys equal to kth are winners
    // keys above the k-th: any order (the sort below fixes it)
    for (int p = tid; p < n; p += NT) {
        const float v = val(p);
        if (sample_key(v) > kth) {
            const unsigned s = atomicAdd(&S.gt, 1u);
            S.win_v[s] = v;
            S.win_p[s] = p;
            S.win_i[s] = idx(p);
        }
    }
    // keys equal to it: the `need` at the lowest positions (contiguous ranges per thread, ranked by
    // a prefix count over the threads)
    const int per = (n + NT - 1) / NT, p0 = min(n, tid * per), p1 = min(n, p0 + per);
    unsigned ties = 0;
    for (int p = p0; p < p1; p++) ties += sample_key(val(p)) == kth;
    unsigned total;
    unsigned rank = block_excl_scan<NT>(S, ties, &total);
    const unsigned first = (unsigned)k - need;
    for (int p = p0; p < p1 && rank < need; p++) {
        const float v = val(p);
        if (sample_key(v) == kth) {
            S.win_v[first + rank] = v;
            S.win_p[first + rank] = p;
            S.win_i[first + rank] = idx(p);
            rank++;
        }
    }
    named_bar_sync(1, NT);
    // order the k winners by (value descending, index ascending)
    if (tid < k) {
        const float v = S.win_v[tid];
        const int i = S.win_i[tid];
        const unsigned kv = sample_key(v);
        int r = 0;
        for (int j = 0; j < k; j++) {
            const unsigned kj = sample_key(S.win_v[j]);
            const int ij = S.win_i[j];
            r += (kj > kv) || (kj == kv && ij < i);
        }
        S.top_v[r] = v;
        S.top_i[r] = i;
    }
    named_bar_sync(1, NT);
    (void)lane;
}

// The sampled token from S.top_v / S.top_i (k candidates), for warp 0; -1 when a candidate is
// not finite. Every lane of warp 0 returns the same value.
KIE_DEV int sample_pick(const SampleScratch &S, int k, float inv_t, float u) {
    const int lane = threadIdx.x & 31;
    const float v0 = S.top_v[0];
    const float v = lane < k ? S.top_v[lane] : v0;
    const bool finite = __all_sync(0xffffffffu, isfinite(v));
    float w = lane < k ? __expf((v - v0) * inv_t) : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
    }
    const float total = __shfl_sync(0xffffffffu, w, k - 1);
    const float r = u * total;
    const unsigned hit = __ballot_sync(0xffffffffu, lane < k && w > r);
    const int pick = hit ? __ffs(hit) - 1 : k - 1;
    return finite ? S.top_i[pick] : -1;
}
