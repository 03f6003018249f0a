// Bf16TrilDiagF32 Hessian codec ("hipfire-calib-data" dataset card, "Hessian storage:
// Bf16TrilDiagF32 (quant_type 130)"): K fp32 diagonal values, then the strict lower
// triangle as bf16 obtained by truncation (fp32 bits >> 16) at index i(i-1)/2 + j.
//
// Encode: for K % 4 == 0 one grid-stride pass of 16-byte payload stores (see
// tril_encode_vec_kernel); otherwise one CTA per row i, whose triangle segment starts at an arbitrary 2-byte offset: a
// scalar head up to the next 16-byte boundary, then 8 values per 16-byte store, then a scalar
// tail.  Loads of H are coalesced fp32 either way.
// Decode ("mirrored on read"): 64 x 64 tiles of the lower triangle; each tile reads its rows'
// triangle segments (coalesced u16), writes H[i, j] row-wise and the mirror H[j, i] through a
// shared-memory transpose so both stores are coalesced.
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

// One pass for K % 4 == 0 (the payload then starts 16-byte aligned) and K <= 46340 (every
// index fits 32 bits).  A warp takes 256 consecutive payload values p = w0 .. w0 + 255: lane l
// loads p = w0 + l + 32 k (k = 0..7), so each load instruction reads 32 consecutive values of
// H (mostly one row: 128 contiguous bytes), truncates them into a shared-memory strip in
// payload order, and then stores 16-byte pieces p = w0 + 256 h + 8 l .. + 7.  The row of w0 is found
// once per warp range; every lane steps from there along the rows.  The diagonal goes in
// 16-byte stores of four values.
constexpr int kEncThreads = 256;
constexpr int kEncRange = 256;  // payload values per warp range (8 loads in flight per lane)

__global__ void __launch_bounds__(kEncThreads) tril_encode_vec_kernel(const float* __restrict__ H, int K,
                                                                      uint8_t* __restrict__ out) {
  __shared__ __align__(16) uint16_t strip[kEncThreads / 32][kEncRange];
  const int lane = threadIdx.x % 32, w = threadIdx.x / 32;
  const int npay = K * (K - 1) / 2;  // payload values
  const int nw = (npay + kEncRange - 1) / kEncRange;  // warp ranges
  uint16_t* my = strip[w];
  uint4* pay4 = reinterpret_cast<uint4*>(out + 4 * static_cast<int64_t>(K));
  uint16_t* pay = reinterpret_cast<uint16_t*>(out + 4 * static_cast<int64_t>(K));
  const int wstride = gridDim.x * (kEncThreads / 32);
  for (int r = blockIdx.x * (kEncThreads / 32) + w; r < nw; r += wstride) {
    const int w0 = kEncRange * r;
    // row of w0: i (i - 1) / 2 <= w0 < i (i + 1) / 2
    int i = static_cast<int>((1.0f + sqrtf(1.0f + 8.0f * static_cast<float>(w0))) * 0.5f);
    while (static_cast<int64_t>(i) * (i - 1) / 2 > w0) --i;
    while (static_cast<int64_t>(i) * (i + 1) / 2 <= w0) ++i;
    int j = w0 - static_cast<int>(static_cast<int64_t>(i) * (i - 1) / 2) + lane;
    while (j >= i && i < K) {
      j -= i;
      ++i;
    }
#pragma unroll
    for (int k = 0; k < kEncRange / 32; ++k) {
      const bool in = w0 + lane + 32 * k < npay;
      my[lane + 32 * k] = in ? static_cast<uint16_t>(__float_as_uint(H[i * K + j]) >> 16) : uint16_t(0);
      j += 32;
      while (j >= i && i < K) {
        j -= i;
        ++i;
      }
    }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < kEncRange / 256; ++h) {
      const int q0 = w0 + 256 * h + 8 * lane;
      if (q0 + 8 <= npay) {
        pay4[q0 / 8] = reinterpret_cast<const uint4*>(my)[32 * h + lane];
      } else {
        for (int e = 0; q0 + e < npay; ++e) pay[q0 + e] = my[256 * h + 8 * lane + e];
      }
    }
    __syncwarp();
  }
  float4* diag4 = reinterpret_cast<float4*>(out);
  for (int u = blockIdx.x * kEncThreads + threadIdx.x; u < K / 4; u += gridDim.x * kEncThreads) {
    const int i = 4 * u;
    diag4[u] = make_float4(H[i * (K + 1)], H[(i + 1) * (K + 1)], H[(i + 2) * (K + 1)], H[(i + 3) * (K + 1)]);
  }
}

hq_status launch_tril_encode(const float* H, int64_t K, uint8_t* out, cudaStream_t s) {
  if (K % 4 == 0 && K <= 46340 && aligned(out, 16)) {
    const int64_t nw = ceil_div(K * (K - 1) / 2, kEncRange);  // warp ranges
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(ceil_div(nw, kEncThreads / 32), 148 * 8));
    tril_encode_vec_kernel<<<static_cast<unsigned>(grid), kEncThreads, 0, s>>>(H, static_cast<int>(K), out);
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
  const int c4 = 4 * (threadIdx.x % 16);
#pragma unroll
  for (int k = 0; k < kDecTile / 16; ++k) {
    const int r = threadIdx.x / 16 + 16 * k;
    const int i = i0 + r;
    const int rowbase = static_cast<int>(static_cast<int64_t>(i) * (i - 1) / 2);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + c4 + q;
      float v = 0.f;
      if (i < K && j < K) {
        if (j < i)
          v = __uint_as_float(static_cast<uint32_t>(tri[rowbase + j]) << 16);
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
    if (i >= K || j >= K) continue;  // K % 4 == 0: a row's 4 columns are all in range or all out
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
      if (i >= K || j >= K) continue;
      *reinterpret_cast<float4*>(H + j * K + i) = make_float4(tile[r4][c], tile[r4 + 1][c], tile[r4 + 2][c], tile[r4 + 3][c]);
    }
  }
}

hq_status launch_tril_decode(const uint8_t* in, int64_t K, float* H, cudaStream_t s) {
  const int64_t nb = ceil_div(K, kDecTile);
  const int64_t tiles = nb * (nb + 1) / 2;
  if (tiles > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  if (K % 4 == 0 && K <= 46340 && aligned(H, 16))
    tril_decode_vec_kernel<<<static_cast<unsigned>(tiles), 256, 0, s>>>(in, static_cast<int>(K), H);
  else
    tril_decode_kernel<<<static_cast<unsigned>(tiles), 256, 0, s>>>(in, K, H);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

}  // namespace hq
