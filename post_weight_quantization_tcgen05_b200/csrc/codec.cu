// Bf16TrilDiagF32 Hessian codec ("hipfire-calib-data" dataset card, "Hessian storage:
// Bf16TrilDiagF32 (quant_type 130)"): K fp32 diagonal values, then the strict lower
// triangle as bf16 obtained by truncation (fp32 bits >> 16) at index i(i-1)/2 + j.
//
// Encode: for K % 4 == 0 one pass over row pairs with float4 loads and 16-byte payload stores
// (tril_encode_pair_kernel); otherwise one CTA per row i, whose triangle segment starts at an
// arbitrary 2-byte offset: a scalar head up to the next 16-byte boundary, then 8 values per
// 16-byte store, then a scalar tail.
// Decode ("mirrored on read"): 64 x 64 tiles of the lower triangle; each tile reads its rows'
// triangle segments (aligned 8-byte words for K % 4 == 0, else u16), writes H[i, j] row-wise and
// the mirror H[j, i] through a shared-memory transpose so both stores are coalesced.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace hq {

__global__ void tril_encode_diag_kernel(const float* __restrict__ H, int64_t K, float* __restrict__ out_diag) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < K;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out_diag[i] = H[i * K + i];
}

__global__ void __launch_bounds__(256) tril_encode_rows_kernel(const float* __restrict__ H, int64_t K,
                                                               uint8_t* __restrict__ out) {
  for (int64_t i = 1 + blockIdx.x; i < K; i += gridDim.x) {
    const float* row = H + i * K;
    const int64_t n = i;
    const int64_t ob = 4 * K + i * (i - 1);  // byte offset of element (i, 0)
    uint16_t* dst = reinterpret_cast<uint16_t*>(out + ob);
    int64_t h = ((16 - (ob & 15)) & 15) >> 1;
    if (h > n) h = n;
    for (int64_t e = threadIdx.x; e < h; e += blockDim.x)
      dst[e] = static_cast<uint16_t>(__float_as_uint(row[e]) >> 16);
    const int64_t nchunks = (n - h) >> 3;
    uint4* dst4 = reinterpret_cast<uint4*>(dst + h);
    for (int64_t c = threadIdx.x; c < nchunks; c += blockDim.x) {
      const float* src = row + h + 8 * c;
      uint32_t b[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) b[u] = __float_as_uint(src[u]) >> 16;
      uint4 v;
      v.x = b[0] | (b[1] << 16);
      v.y = b[2] | (b[3] << 16);
      v.z = b[4] | (b[5] << 16);
      v.w = b[6] | (b[7] << 16);
      dst4[c] = v;
    }
    for (int64_t e = h + 8 * nchunks + threadIdx.x; e < n; e += blockDim.x)
      dst[e] = static_cast<uint16_t>(__float_as_uint(row[e]) >> 16);
  }
}

// One pass for K % 4 == 0 (16-byte aligned rows of H and payload start) and K <= 46340 (payload
// indices fit 32 bits), balanced by rows: CTA p takes rows 1 + p and K - 1 - p (K values between
// them).  A warp takes 512-value chunks of a row: each lane loads four float4 of H (512
// contiguous bytes per load instruction), truncates them into the warp's shared-memory strip at
// their payload positions (the strip starts at the 16-byte boundary at or below the chunk's
// first payload value), and the chunk's payload piece is then stored as aligned 16-byte words,
// its unaligned head and tail (shared with the neighbouring pieces) as 2-byte stores.  CTA p
// also writes diagonal entries 4p .. 4p + 3.
constexpr int kEncChunk = 512;                   // values per warp chunk (4 float4 per lane)
constexpr int kEncStrip = kEncChunk + 16;        // strip length in u16 (alignment slack)
constexpr int kEncPairThreads = 128;             // 4 warps: about 3 chunks each per row pair

__global__ void __launch_bounds__(kEncPairThreads) tril_encode_pair_kernel(const float* __restrict__ H, int K,
                                                                           uint8_t* __restrict__ out) {
  __shared__ __align__(16) uint16_t strip[kEncPairThreads / 32][kEncStrip];
  const int lane = threadIdx.x % 32, w = threadIdx.x / 32;
  uint16_t* my = strip[w];
  uint16_t* pay = reinterpret_cast<uint16_t*>(out + 4 * static_cast<int64_t>(K));
  uint4* pay4 = reinterpret_cast<uint4*>(pay);
  const int p = blockIdx.x;
  const int ra = 1 + p, rb = K - 1 - p;
  const int na = (ra + kEncChunk - 1) / kEncChunk;
  const int nb = rb > ra ? (rb + kEncChunk - 1) / kEncChunk : 0;
  for (int t = w; t < na + nb; t += kEncPairThreads / 32) {
    const int i = t < na ? ra : rb;
    const int c0 = (t < na ? t : t - na) * kEncChunk;
    const int len = min(kEncChunk, i - c0);  // values of row i in this chunk
    const int P0 = i * (i - 1) / 2 + c0;     // payload index of (i, c0)
    const int base = P0 & ~7;
    const float* src = H + static_cast<int64_t>(i) * K + c0;
    float4 v[kEncChunk / 128];
#pragma unroll
    for (int u = 0; u < kEncChunk / 128; ++u) {
      const int c = 4 * lane + 128 * u;
      v[u] = c < len ? reinterpret_cast<const float4*>(src)[c / 4] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kEncChunk / 128; ++u) {
      const int c = 4 * lane + 128 * u;
      const int d = P0 - base + c;
      const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (c + q < len && HQ_IN_BOUNDS(d + q < kEncStrip)) my[d + q] = static_cast<uint16_t>(__float_as_uint(f[q]) >> 16);
    }
    __syncwarp();
    const int P1 = P0 + len;
    const int A0 = (P0 + 7) & ~7, A1 = P1 & ~7;
    for (int a = A0 + 8 * lane; a + 8 <= A1; a += 256)
      if (HQ_IN_BOUNDS(a + 8 <= K * (K - 1) / 2 && a - base + 8 <= kEncStrip))
        pay4[a / 8] = *reinterpret_cast<const uint4*>(my + (a - base));
    const int h1 = min(A0, P1);
    if (P0 + lane < h1 && HQ_IN_BOUNDS(P0 + lane < K * (K - 1) / 2)) pay[P0 + lane] = my[P0 + lane - base];
    const int t0 = max(A1, A0);
    if (t0 + lane < P1 && HQ_IN_BOUNDS(t0 + lane < K * (K - 1) / 2)) pay[t0 + lane] = my[t0 + lane - base];
    __syncwarp();
  }
  if (4 * p < K) {  // diagonal entries 4p .. 4p + 3 (K % 4 == 0)
    float4* diag4 = reinterpret_cast<float4*>(out);
    if (threadIdx.x == 0) {
      const int i = 4 * p;
      diag4[p] = make_float4(H[static_cast<int64_t>(i) * (K + 1)], H[static_cast<int64_t>(i + 1) * (K + 1)],
                             H[static_cast<int64_t>(i + 2) * (K + 1)], H[static_cast<int64_t>(i + 3) * (K + 1)]);
    }
  }
}

hq_status launch_tril_encode(const float* H, int64_t K, uint8_t* out, cudaStream_t s) {
  if (K % 4 == 0 && K <= 46340 && aligned(out, 16) && aligned(H, 16)) {
    // row pairs, and at least K / 4 CTAs for the diagonal
    const int64_t grid = std::max<int64_t>(K / 2, K / 4);
    tril_encode_pair_kernel<<<static_cast<unsigned>(grid), kEncPairThreads, 0, s>>>(H, static_cast<int>(K), out);
    HQ_LAUNCH_CHECK();
    return HQ_OK;
  }
  const int dg = static_cast<int>(ceil_div(K, 256) < 4096 ? ceil_div(K, 256) : 4096);
  tril_encode_diag_kernel<<<dg, 256, 0, s>>>(H, K, reinterpret_cast<float*>(out));
  HQ_LAUNCH_CHECK();
  if (K > 1) {
    const int64_t rows = K - 1;
    const int grid = static_cast<int>(rows < 65535 ? rows : 65535);
    tril_encode_rows_kernel<<<grid, 256, 0, s>>>(H, K, out);
    HQ_LAUNCH_CHECK();
  }
  return HQ_OK;
}

constexpr int kDecTile = 64;

__global__ void __launch_bounds__(256) tril_decode_kernel(const uint8_t* __restrict__ in, int64_t K,
                                                          float* __restrict__ H) {
  __shared__ float tile[kDecTile][kDecTile + 1];
  int64_t t = blockIdx.x;
  int64_t bi = static_cast<int64_t>((sqrt(8.0 * static_cast<double>(t) + 1.0) - 1.0) * 0.5);
  while (bi * (bi + 1) / 2 > t) --bi;
  while ((bi + 1) * (bi + 2) / 2 <= t) ++bi;
  const int64_t bj = t - bi * (bi + 1) / 2;
  const int64_t i0 = bi * kDecTile, j0 = bj * kDecTile;
  const float* diag = reinterpret_cast<const float*>(in);
  const uint16_t* tri = reinterpret_cast<const uint16_t*>(in + 4 * K);
  // gather: tile[r][c] = value of (i0 + r, j0 + c) for the lower triangle incl. diagonal
  for (int e = threadIdx.x; e < kDecTile * kDecTile; e += 256) {
    const int r = e / kDecTile, c = e % kDecTile;
    const int64_t i = i0 + r, j = j0 + c;
    float v = 0.f;
    if (i < K && j < K) {
      if (j < i)
        v = __uint_as_float(static_cast<uint32_t>(tri[i * (i - 1) / 2 + j]) << 16);
      else if (j == i)
        v = diag[i];
    }
    tile[r][c] = v;
  }
  __syncthreads();
  // row-wise store of the lower part (and, on diagonal tiles, of the mirrored upper part)
  for (int e = threadIdx.x; e < kDecTile * kDecTile; e += 256) {
    const int r = e / kDecTile, c = e % kDecTile;
    const int64_t i = i0 + r, j = j0 + c;
    if (i >= K || j >= K) continue;
    if (bi == bj)
      H[i * K + j] = (c <= r) ? tile[r][c] : tile[c][r];
    else
      H[i * K + j] = tile[r][c];
  }
  if (bi != bj) {
    // mirror: H[j, i] for the tile's (i, j): row j0 + c of H, columns i0 + r
    for (int e = threadIdx.x; e < kDecTile * kDecTile; e += 256) {
      const int c = e / kDecTile, r = e % kDecTile;
      const int64_t i = i0 + r, j = j0 + c;
      if (i >= K || j >= K) continue;
      H[j * K + i] = tile[r][c];
    }
  }
}

// K % 4 == 0 and K <= 46340 (32-bit indices): the same tiles with 16-byte stores.  Thread t gathers 4 consecutive columns of
// rows t / 16 + 16 k and stores 4 consecutive floats of a row of H (lower part, row-wise) and
// of a row of the mirror (H[j, i0 + r .. r + 3], read down a column of the tile).
__global__ void __launch_bounds__(256) tril_decode_vec_kernel(const uint8_t* __restrict__ in, int K,
                                                              float* __restrict__ H) {
  __shared__ float tile[kDecTile][kDecTile + 1];
  const int t = blockIdx.x;
  int bi = static_cast<int>((sqrtf(8.0f * static_cast<float>(t) + 1.0f) - 1.0f) * 0.5f);
  while (bi * (bi + 1) / 2 > t) --bi;
  while ((bi + 1) * (bi + 2) / 2 <= t) ++bi;
  const int bj = t - bi * (bi + 1) / 2;
  const int i0 = bi * kDecTile, j0 = bj * kDecTile;
  const float* diag = reinterpret_cast<const float*>(in);
  const uint16_t* tri = reinterpret_cast<const uint16_t*>(in + 4 * static_cast<int64_t>(K));
  const uint2* tri8 = reinterpret_cast<const uint2*>(tri);  // 8-byte words (the payload starts 16-byte aligned)
  const int npay = K * (K - 1) / 2;
  const int c4 = 4 * (threadIdx.x % 16);
  const int hl = threadIdx.x % 16;  // lane within the half-warp that owns a row
  // A row's 64 values start at payload index s = i(i-1)/2 + j0, 2-byte aligned: lane hl loads the
  // aligned word holding values s - m + 4 hl .. + 3 (m = s mod 4) and takes its four values from
  // that word and the next lane's (lane 15 loads the 17th word itself).  Words that would reach
  // past the payload are read value by value.
  auto word = [&](int x) -> uint64_t {
    if (4 * x + 4 <= npay) {
      const uint2 v = tri8[x];
      return static_cast<uint64_t>(v.x) | (static_cast<uint64_t>(v.y) << 32);
    }
    uint64_t v = 0;
    for (int q = 0; q < 4; ++q)
      if (4 * x + q < npay) v |= static_cast<uint64_t>(tri[4 * x + q]) << (16 * q);
    return v;
  };
#pragma unroll
  for (int k = 0; k < kDecTile / 16; ++k) {
    const int r = threadIdx.x / 16 + 16 * k;
    const int i = i0 + r;
    const int ncol = i < K ? min(i, j0 + kDecTile) - j0 : 0;  // payload values of this row in the tile
    uint64_t own = 0, nxt = 0;
    int m = 0;
    if (ncol > 0) {
      const int sidx = i * (i - 1) / 2 + j0;
      m = sidx & 3;
      const int wb = (sidx - m) / 4;
      if (4 * hl < m + ncol) own = word(wb + hl);
      if (hl == 15 && m + ncol > 64) nxt = word(wb + 16);
    }
    const uint64_t from_next = __shfl_down_sync(0xffffffffu, own, 1, 16);
    if (hl != 15) nxt = from_next;
    // values m + 4 hl .. m + 4 hl + 3 of the window = bits 16 m .. of (nxt : own)
    const uint64_t vals = m == 0 ? own : ((own >> (16 * m)) | (nxt << (64 - 16 * m)));
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + c4 + q;
      float v = 0.f;
      if (i < K && j < K) {
        if (j < i)
          v = __uint_as_float(static_cast<uint32_t>((vals >> (16 * q)) & 0xFFFFu) << 16);
        else if (j == i)
          v = diag[i];
      }
      tile[r][c4 + q] = v;
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kDecTile / 16; ++k) {
    const int r = threadIdx.x / 16 + 16 * k;
    const int64_t i = i0 + r, j = j0 + c4;
    if (i >= K || j >= K || !HQ_IN_BOUNDS(j + 3 < K)) continue;  // K % 4 == 0: a row's 4 columns are all in range or all out
    float4 o;
    if (bi == bj) {
      o.x = (c4 + 0 <= r) ? tile[r][c4 + 0] : tile[c4 + 0][r];
      o.y = (c4 + 1 <= r) ? tile[r][c4 + 1] : tile[c4 + 1][r];
      o.z = (c4 + 2 <= r) ? tile[r][c4 + 2] : tile[c4 + 2][r];
      o.w = (c4 + 3 <= r) ? tile[r][c4 + 3] : tile[c4 + 3][r];
    } else {
      o = make_float4(tile[r][c4], tile[r][c4 + 1], tile[r][c4 + 2], tile[r][c4 + 3]);
    }
    *reinterpret_cast<float4*>(H + i * K + j) = o;
  }
  if (bi != bj) {
    // mirror: H[j0 + c, i0 + r4 .. r4 + 3] = tile[r4 .. r4 + 3][c]
#pragma unroll
    for (int k = 0; k < kDecTile / 16; ++k) {
      const int c = threadIdx.x / 16 + 16 * k, r4 = c4;
      const int64_t j = j0 + c, i = i0 + r4;
      if (i >= K || j >= K || !HQ_IN_BOUNDS(i + 3 < K)) continue;
      *reinterpret_cast<float4*>(H + j * K + i) = make_float4(tile[r4][c], tile[r4 + 1][c], tile[r4 + 2][c], tile[r4 + 3][c]);
    }
  }
}


hq_status launch_tril_decode(const uint8_t* in, int64_t K, float* H, cudaStream_t s) {
  const int64_t nb = ceil_div(K, kDecTile);
  const int64_t tiles = nb * (nb + 1) / 2;
  if (tiles > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  if (K % 4 == 0 && K <= 46340 && aligned(H, 16) && aligned(in, 8))
    tril_decode_vec_kernel<<<static_cast<unsigned>(tiles), 256, 0, s>>>(in, static_cast<int>(K), H);
  else
    tril_decode_kernel<<<static_cast<unsigned>(tiles), 256, 0, s>>>(in, K, H);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

}  // namespace hq
