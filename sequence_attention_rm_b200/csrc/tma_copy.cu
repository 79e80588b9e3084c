// Bit-exact layout transforms through the TMA unit.
//
// The Ulysses repack and the token permutations move whole runs of bytes
// between two orders of the same tensor.  Both orders are written as 5-D
// tensor maps over the same box: the source map and the destination map have
// the same dimensions and differ only in their strides (and, for the zigzag
// chunks, in one coordinate), so a box loaded from the source view lands in
// shared memory already in destination order and is stored back with one
// TMA store.  One thread per CTA drives a ring of two 32 KB stages (the next
// load is in flight while the current tile is stored); three CTAs fit on an
// SM.  The grid has one CTA per tile, handed out as SMs free up: on B200 the
// 2 x 1 GiB repack ran at 6.86 TB/s (1.05 of the measured copy rate) and the
// 1 GiB striped permute at 6.52, against 6.17 / 6.09 for one wave of three
// CTAs per SM that loop over the tiles (2, 4, 8, 16 tiles per CTA fell in
// between, in that order); one CTA per SM with a six-stage ring reached 5.8,
// 16 KB stages 3.8.
// Every wait is bounded; on a timeout the kernel records it in the status
// word, drains its own copies and returns.
#include <climits>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace rm {

rm_status encode_copy_map(CUtensorMap* map, const void* ptr, int esize, const int64_t (&dims)[5],
                          const int64_t (&strides)[4], const int (&box)[5]);
long long tc_wait_limit();
unsigned int* status_word();

namespace {

using namespace tc;

constexpr int kStages = 2;
constexpr int kStageBytes = 32 << 10;
constexpr int kAhead = kStages - 1;  // loads in flight ahead of the store
constexpr int kCtasPerSm = 3;

struct TmaCopyParams {
  int tiles[5];   // tiles along each dimension
  int box[5];
  int64_t total;  // product of tiles
  int remap;      // 0: same coordinates; 1 / 2: zigzag chunk <-> rank slot on dimension 3
  int P;
  uint32_t tile_bytes;
  unsigned int* status;
  long long wait_limit;
};

__device__ __forceinline__ void tma_store_5d(const CUtensorMap* map, const void* smem_src, int c0,
                                             int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4, %5}], [%6];" ::
          "l"(reinterpret_cast<uint64_t>(map)),
      "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_u32(smem_src))
      : "memory");
}
// Wait until at most the most recent bulk group is still reading shared memory.
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

__global__ void __launch_bounds__(32, kCtasPerSm)
    tma_copy_kernel(const __grid_constant__ CUtensorMap src, const __grid_constant__ CUtensorMap dst,
                    const TmaCopyParams p) {
  // stages, then the barriers, all in dynamic shared memory (no static
  // shared memory, so the stages start at the base of the CTA's window)
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  if (threadIdx.x != 0) return;
  if (smem_u32(smem) & 127u) {  // TMA boxes need a 128-byte aligned destination
    report_status(p.status, kStatusSmemAlign);
    return;
  }
  for (int s = 0; s < kStages; ++s) mbar_init(bars + s, 1);
  fence_barrier_init();
  prefetch_tmap(&src);
  prefetch_tmap(&dst);
  const int64_t first = blockIdx.x, stride = gridDim.x;
  const int64_t mine = p.total > first ? (p.total - first + stride - 1) / stride : 0;
  auto coords = [&](int64_t k, int (&c)[5]) {
    int64_t t = first + k * stride;
#pragma unroll
    for (int d = 0; d < 5; ++d) {
      const int64_t q = t / p.tiles[d];
      c[d] = (int)(t - q * p.tiles[d]) * p.box[d];
      t = q;
    }
  };
  auto load = [&](int64_t k) {
    int c[5];
    coords(k, c);
    const int st = (int)(k % kStages);
    mbar_arrive_expect_tx(bars + st, p.tile_bytes);
    tma_load_5d(smem + st * kStageBytes, &src, bars + st, c[0], c[1], c[2], c[3], c[4]);
  };
  int64_t issued = 0;
  for (; issued < mine && issued < kAhead; ++issued) load(issued);
  int64_t k = 0;
  for (; k < mine; ++k) {
    const int st = (int)(k % kStages);
    if (!mbar_wait(bars + st, (uint32_t)((k / kStages) & 1), p.wait_limit, p.status)) break;
    int c[5];
    coords(k, c);
    if (p.remap == 1)  // global chunk q -> slot 2r + half of rank r
      c[3] = c[3] < p.P ? 2 * c[3] : 2 * (2 * p.P - 1 - c[3]) + 1;
    else if (p.remap == 2)  // slot 2r + half -> global chunk
      c[3] = (c[3] & 1) ? 2 * p.P - 1 - (c[3] >> 1) : (c[3] >> 1);
    tma_store_5d(&dst, smem + st * kStageBytes, c[0], c[1], c[2], c[3], c[4]);
    bulk_commit();
    if (issued < mine) {
      // the stage of load `issued` was last stored from by tile issued - kStages = k - 1
      bulk_wait_read_1();
      load(issued);
      ++issued;
    }
  }
  // drain: loads issued but not consumed (after a timeout), then every store
  for (int64_t j = k; j < issued; ++j)
    mbar_wait(bars + (int)(j % kStages), (uint32_t)((j / kStages) & 1), p.wait_limit, p.status);
  bulk_wait_all();
}

bool fits(const int (&box)[5], int esize) {
  int64_t bytes = esize;
  for (int d = 0; d < 5; ++d) {
    if (box[d] < 1 || box[d] > 256) return false;
    bytes *= box[d];
  }
  return (box[0] * esize) % 16 == 0 && bytes <= kStageBytes;
}

// Runs the copy if both views encode; returns false (nothing launched) when the
// shapes are outside what the TMA path handles.
bool run_copy(const char* name, const void* in, void* out, int esize, const int64_t (&dims)[5],
              const int64_t (&src_strides)[4], const int64_t (&dst_strides)[4],
              const int (&box)[5], int remap, int P, cudaStream_t stream, cudaError_t* err) {
  if (!fits(box, esize) || ((uintptr_t)in | (uintptr_t)out) % 16) return false;
  for (int d = 0; d < 4; ++d)
    if (src_strides[d] % 16 || dst_strides[d] % 16) return false;
  CUtensorMap ms, md;
  if (encode_copy_map(&ms, in, esize, dims, src_strides, box) != RM_OK ||
      encode_copy_map(&md, out, esize, dims, dst_strides, box) != RM_OK)
    return false;
  TmaCopyParams p;
  p.total = 1;
  p.tile_bytes = (uint32_t)esize;
  for (int d = 0; d < 5; ++d) {
    p.box[d] = box[d];
    p.tiles[d] = (int)((dims[d] + box[d] - 1) / box[d]);
    p.total *= p.tiles[d];
    p.tile_bytes *= (uint32_t)box[d];
  }
  p.remap = remap;
  p.P = P;
  p.status = status_word();
  p.wait_limit = tc_wait_limit();
  if (p.total == 0) {
    *err = cudaSuccess;
    return true;
  }
  const int smem_bytes = kStages * kStageBytes + kStages * 8;
  if (cudaFuncSetAttribute(tma_copy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_bytes) != cudaSuccess)
    return false;
  // one CTA per tile (the kernel's stride loop covers any tiles past the cap)
  const int64_t grid = p.total < INT_MAX ? p.total : INT_MAX;
  ProfScope ps(name, stream);
  tma_copy_kernel<<<(unsigned)grid, 32, smem_bytes, stream>>>(ms, md, p);
  *err = cudaGetLastError();
  return true;
}

}  // namespace

// Ulysses repack as a TMA copy: the tensor is runs of E = (H/P)*d elements,
// [n][r][E] in sequence-sharded order (n = s*L + t over all P*L tokens, r the
// head group) and [r][n][E] in head-sharded order; a box covers all P groups
// of k consecutive tokens.
bool tma_seq_head_repack(int esize, int P, int64_t n_local, int H, int d, int head_to_seq,
                         const void* in, void* out, cudaStream_t stream, cudaError_t* err) {
  const int64_t E = (int64_t)(H / P) * d, ntot = (int64_t)P * n_local;
  if (E > 256 || P > 256) return false;
  const int64_t run = E * esize;
  int k = (int)(kStageBytes / (run * P));
  if (k < 1) return false;
  if (k > 256) k = 256;
  const int64_t dims[5] = {E, ntot, P, 1, 1};
  const int64_t seq[4] = {P * run, run, ntot * P * run, ntot * P * run};  // [n][r][E]
  const int64_t head[4] = {run, ntot * run, ntot * P * run, ntot * P * run};  // [r][n][E]
  const int box[5] = {(int)E, k, P, 1, 1};
  return run_copy("seq_head_repack", in, out, esize, dims, head_to_seq ? head : seq,
                  head_to_seq ? seq : head, box, 0, P, stream, err);
}

// Token permutation global <-> rank-major of [B, N, H, d] as a TMA copy.
// Rows are R = H*d elements, split as (d, H) so that each box dimension stays
// within 256 elements.  Striped: global row j*P + r <-> rank-major r*L + j,
// a pure stride swap of the (j, r) dimensions.  Zigzag: chunks of C rows;
// global chunk q <-> rank slot (r, half) by a coordinate remap on dimension 3.
// Contiguous: the identity.
bool tma_layout_permute(int esize, int B, int64_t N, int H, int d, int layout, int P,
                        int inverse, const void* in, void* out, cudaStream_t stream,
                        cudaError_t* err) {
  if (d > 256 || H > 256) return false;
  const int64_t row = (int64_t)H * d * esize;
  const int64_t L = N / P;
  int k = (int)(kStageBytes / row);  // rows per box
  if (k < 1) return false;
  if (k > 256) k = 256;
  if (layout == RM_LAYOUT_STRIPED) {
    const int64_t dims[5] = {d, H, L, P, B};
    const int64_t glob[4] = {(int64_t)d * esize, P * row, row, N * row};  // row j*P + r
    const int64_t rank[4] = {(int64_t)d * esize, row, L * row, N * row};  // row r*L + j
    const int box[5] = {d, H, k, 1, 1};
    return run_copy("layout_permute", in, out, esize, dims, inverse ? rank : glob,
                    inverse ? glob : rank, box, 0, P, stream, err);
  }
  if (layout == RM_LAYOUT_ZIGZAG) {
    const int64_t C = N / (2 * P);
    const int64_t dims[5] = {d, H, C, 2 * P, B};
    const int64_t str[4] = {(int64_t)d * esize, row, C * row, N * row};  // chunk or slot c*C
    const int box[5] = {d, H, k, 1, 1};
    return run_copy("layout_permute", in, out, esize, dims, str, str, box, inverse ? 2 : 1, P,
                    stream, err);
  }
  const int64_t dims[5] = {d, H, N, 1, B};
  const int64_t str[4] = {(int64_t)d * esize, row, N * row, N * row};
  const int box[5] = {d, H, k, 1, 1};
  return run_copy("layout_permute", in, out, esize, dims, str, str, box, 0, P, stream, err);
}

}  // namespace rm
