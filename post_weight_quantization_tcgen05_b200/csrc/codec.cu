// Bf16TrilDiagF32 Hessian codec ("hipfire-calib-data" dataset card, "Hessian storage:
// Bf16TrilDiagF32 (quant_type 130)"): K fp32 diagonal values, then the strict lower
// triangle as bf16 obtained by truncation (fp32 bits >> 16) at index i(i-1)/2 + j.
//
// Encode: one CTA per row i; the row's triangle segment starts at an arbitrary 2-byte
// offset, so each CTA writes a scalar head up to the next 16-byte boundary, then 8 values per
// 16-byte store, then a scalar tail.  Loads of H's row are coalesced fp32.
// Decode ("mirrored on read"): 64 x 64 tiles of the lower triangle; each tile reads its rows'
// triangle segments (coalesced u16), writes H[i, j] row-wise and the mirror H[j, i] through a
// shared-memory transpose so both stores are coalesced.
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

hq_status launch_tril_encode(const float* H, int64_t K, uint8_t* out, cudaStream_t s) {
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

hq_status launch_tril_decode(const uint8_t* in, int64_t K, float* H, cudaStream_t s) {
  const int64_t nb = ceil_div(K, kDecTile);
  const int64_t tiles = nb * (nb + 1) / 2;
  if (tiles > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  tril_decode_kernel<<<static_cast<unsigned>(tiles), 256, 0, s>>>(in, K, H);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

}  // namespace hq
