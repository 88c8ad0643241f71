// Scan locality of an index map over a T x H x W latent grid (news article, method section, Rotary Major
// Scan paragraphs; "LinGen：基于Mamba机制的线性复杂度高清长视频生成框架", 功能特色 / RMS): the sum, count and
// maximum over all pairs of grid-adjacent tokens of their distance in the scanned sequence.  The pages
// claim the alternating scan orders bring the mean of that distance down to the level of Zigzag and
// Hilbert scans; this kernel measures it for the maps:
//   0..3  the Rotary Major Scan orders;
//   4     Zigzag: the 3D boustrophedon (w fastest, reversing on every (t, h) line; h reversing on every t
//         plane; t ascending);
//   5     Hilbert: cubes of side H = W (a power of two) stacked along t, each traversed by the 3D Hilbert
//         curve (transposed-index construction of Skilling, "Programming the Hilbert curve", 2004);
//   6     the rotation of the four orders: per pair the smallest distance over the four orders.
#pragma once
#include "common.cuh"

namespace mate {

__device__ __forceinline__ long long zigzag_pos(int t, int h, int w, int H, int W) {
  const int j = (t & 1) ? H - 1 - h : h;            // lines of plane t visited before (t, h)
  const long long line = static_cast<long long>(t) * H + j;
  const int ww = (line & 1) ? W - 1 - w : w;
  return line * W + ww;
}

__device__ __forceinline__ long long hilbert_pos(int t, int h, int w, int S, int bits) {
  const int cube = t / S;
  unsigned X[3] = {static_cast<unsigned>(t - cube * S), static_cast<unsigned>(h), static_cast<unsigned>(w)};
  const unsigned M = 1u << (bits - 1);
  for (unsigned Q = M; Q > 1; Q >>= 1) {       // undo the excess work of the reflections and exchanges
    const unsigned P = Q - 1;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      if (X[i] & Q) {
        X[0] ^= P;
      } else {
        const unsigned tt = (X[0] ^ X[i]) & P;
        X[0] ^= tt;
        X[i] ^= tt;
      }
    }
  }
  X[1] ^= X[0];                                  // Gray encode
  X[2] ^= X[1];
  unsigned tt = 0;
  for (unsigned Q = M; Q > 1; Q >>= 1)
    if (X[2] & Q) tt ^= Q - 1;
#pragma unroll
  for (int i = 0; i < 3; ++i) X[i] ^= tt;
  unsigned long long idx = 0;                    // interleave the transposed bits, most significant first
  for (int b = bits - 1; b >= 0; --b)
#pragma unroll
    for (int i = 0; i < 3; ++i) idx = (idx << 1) | ((X[i] >> b) & 1u);
  return static_cast<long long>(cube) * S * S * S + static_cast<long long>(idx);
}

__device__ __forceinline__ long long map_pos(int kind, int t, int h, int w, int T, int H, int W, int bits) {
  if (kind <= 3) return raster_to_scan((t * H + h) * W + w, T, H, W, kind);
  if (kind == 4) return zigzag_pos(t, h, w, H, W);
  return hilbert_pos(t, h, w, H, bits);
}

__device__ __forceinline__ long long pair_dist(int kind, int t, int h, int w, int t2, int h2, int w2, int T, int H,
                                               int W, int bits) {
  if (kind == 6) {
    long long best = LLONG_MAX;
#pragma unroll
    for (int o = 0; o < 4; ++o) {
      const long long d = llabs(map_pos(o, t, h, w, T, H, W, bits) - map_pos(o, t2, h2, w2, T, H, W, bits));
      best = d < best ? d : best;
    }
    return best;
  }
  return llabs(map_pos(kind, t, h, w, T, H, W, bits) - map_pos(kind, t2, h2, w2, T, H, W, bits));
}

// One thread per token: the pairs with its +1 neighbour along t, h and w.  out[0] += sum of distances,
// out[1] += pairs, out[2] = max(out[2], largest distance); out must be zero on entry.
__global__ void scan_locality_kernel(int T, int H, int W, int kind, int bits, unsigned long long* out) {
  const long long n = static_cast<long long>(T) * H * W;
  unsigned long long sum = 0, pairs = 0, mx = 0;
  for (long long r = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; r < n;
       r += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int w = static_cast<int>(r % W), h = static_cast<int>((r / W) % H), t = static_cast<int>(r / (W * H));
    const int nb[3][3] = {{t + 1, h, w}, {t, h + 1, w}, {t, h, w + 1}};
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      if (nb[a][0] < T && nb[a][1] < H && nb[a][2] < W) {
        const unsigned long long d =
            static_cast<unsigned long long>(pair_dist(kind, t, h, w, nb[a][0], nb[a][1], nb[a][2], T, H, W, bits));
        sum += d;
        pairs += 1;
        mx = d > mx ? d : mx;
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    sum += __shfl_down_sync(0xffffffffu, sum, off);
    pairs += __shfl_down_sync(0xffffffffu, pairs, off);
    const unsigned long long o = __shfl_down_sync(0xffffffffu, mx, off);
    mx = o > mx ? o : mx;
  }
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(&out[0], sum);
    atomicAdd(&out[1], pairs);
    atomicMax(&out[2], mx);
  }
}

}  // namespace mate
