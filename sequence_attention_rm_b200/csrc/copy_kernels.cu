// Bit-exact layout transforms: global <-> rank-major token permutation and
// the Ulysses sequence <-> head repack.  Both are row gathers of contiguous
// byte runs, done with 16-byte vector loads/stores where the run length and
// the pointers allow it.  HBM-bound: algorithmic traffic is one read and one
// write of the tensor.
#include "common.cuh"
#include "internal.h"

namespace rm {

// TMA path of the two transforms (tma_copy.cu); false when the shape is
// outside it (odd row sizes, misaligned pointers), and the gather kernel runs.
bool tma_seq_head_repack(int esize, int P, int64_t n_local, int H, int d, int head_to_seq,
                         const void* in, void* out, cudaStream_t stream, cudaError_t* err);
bool tma_layout_permute(int esize, int B, int64_t N, int H, int d, int layout, int P,
                        int inverse, const void* in, void* out, cudaStream_t stream,
                        cudaError_t* err);

namespace {

// Copies `rows` runs of `run_vecs` vectors.  Run i goes from src + so(i) to
// dst + dof(i) (byte offsets from the map).  The work is cut into items of
// one run's 32-vector chunk, one vector per lane; a warp takes K consecutive
// items per pass and keeps all K loads in flight before the stores.  The map
// (integer divisions) is evaluated once per item by lane u of the warp and
// broadcast with shuffles, so its cost is shared by the 32 lanes.
template <typename VEC, int K, typename Map>
__global__ void __launch_bounds__(256, 4) gather_runs_kernel(const char* __restrict__ src,
                                                          char* __restrict__ dst, int64_t rows,
                                                          int run_vecs, Map map) {
  static_assert(K <= 32, "one item per lane for the map evaluation");
  const int lane = threadIdx.x & 31;
  const int chunks = (run_vecs + 31) >> 5;
  const int64_t items = rows * chunks;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t base = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * K;
       base < items; base += nwarps * K) {
    // lane u < K evaluates item base + u
    int64_t my_so = 0, my_dof = 0;
    int my_v0 = 0;
    {
      const int64_t it = base + (lane < K ? lane : 0);
      if (it < items) {
        const int64_t row = chunks == 1 ? it : it / chunks;
        my_v0 = (int)(it - row * chunks) * 32;
        map(row, my_so, my_dof);
      }
    }
    VEC buf[K];
#pragma unroll
    for (int u = 0; u < K; ++u) {
      const int64_t so = __shfl_sync(0xffffffffu, my_so, u);
      const int v = __shfl_sync(0xffffffffu, my_v0, u) + lane;
      if (base + u < items && v < run_vecs)
        buf[u] = __ldcs(reinterpret_cast<const VEC*>(src + so) + v);
    }
#pragma unroll
    for (int u = 0; u < K; ++u) {
      const int64_t dof = __shfl_sync(0xffffffffu, my_dof, u);
      const int v = __shfl_sync(0xffffffffu, my_v0, u) + lane;
      if (base + u < items && v < run_vecs)
        __stcs(reinterpret_cast<VEC*>(dst + dof) + v, buf[u]);
    }
  }
}

// Row map of the token permutation: output row (b, r*L + j) <- input row
// (b, pos(r, j)) (forward) or the reverse.
struct PermuteMap {
  static constexpr const char* kName = "layout_permute";
  LayoutMap lay;
  int64_t N;
  int64_t row_bytes;
  int inverse;
  __device__ __forceinline__ void operator()(int64_t row, int64_t& so, int64_t& dof) const {
    int64_t b = row / N;
    int64_t n = row - b * N;           // rank-major index
    int r = (int)(n / lay.L);
    int64_t j = n - (int64_t)r * lay.L;
    int64_t g = lay.pos(r, j);         // global index
    int64_t rm_off = (b * N + n) * row_bytes;
    int64_t gl_off = (b * N + g) * row_bytes;
    if (inverse) { so = rm_off; dof = gl_off; }
    else { so = gl_off; dof = rm_off; }
  }
};

// Run map of the repack, seen as [Ntot][P][run] <-> [P][Ntot][run] with
// Ntot = P * N_local and run = (H/P) * d elements:
//   seq -> head: out[r][n] <- in[n][r];   head -> seq: out[n][r] <- in[r][n].
struct RepackMap {
  static constexpr const char* kName = "seq_head_repack";
  int64_t ntot;
  int P;
  int64_t run_bytes;
  int head_to_seq;
  __device__ __forceinline__ void operator()(int64_t row, int64_t& so, int64_t& dof) const {
    // row enumerates the destination runs in destination order
    if (!head_to_seq) {
      int64_t r = row / ntot, n = row - r * ntot;
      so = (n * P + r) * run_bytes;
      dof = row * run_bytes;
    } else {
      int64_t n = row / P, r = row - n * P;
      so = (r * ntot + n) * run_bytes;
      dof = row * run_bytes;
    }
  }
};

template <typename Map>
cudaError_t launch_gather(const void* src, void* dst, int64_t rows, int64_t run_bytes, Map map,
                          cudaStream_t stream) {
  if (rows == 0 || run_bytes == 0) return cudaSuccess;
  const int threads = 256;
  constexpr int K = 8;
  const uintptr_t a = (uintptr_t)src | (uintptr_t)dst;
  const int vsz = (run_bytes % 16 == 0 && a % 16 == 0) ? 16 : (run_bytes % 4 == 0 && a % 4 == 0) ? 4 : 2;
  const int64_t run_vecs = run_bytes / vsz;
  const int64_t items = rows * ((run_vecs + 31) / 32);
  const int64_t warps_cap = (int64_t)num_sms() * 4 * (threads / 32);  // 4 resident blocks per SM
  const int64_t warps_need = (items + K - 1) / K;
  const int64_t warps = warps_need < warps_cap ? warps_need : warps_cap;
  const int blocks = (int)((warps + (threads / 32) - 1) / (threads / 32));
  ProfScope ps(Map::kName, stream);
  if (vsz == 16)
    gather_runs_kernel<uint4, K, Map><<<blocks, threads, 0, stream>>>(
        (const char*)src, (char*)dst, rows, (int)run_vecs, map);
  else if (vsz == 4)
    gather_runs_kernel<uint32_t, K, Map><<<blocks, threads, 0, stream>>>(
        (const char*)src, (char*)dst, rows, (int)run_vecs, map);
  else
    gather_runs_kernel<uint16_t, K, Map><<<blocks, threads, 0, stream>>>(
        (const char*)src, (char*)dst, rows, (int)run_vecs, map);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_layout_permute(int esize, int B, int64_t N, int H, int d, int layout, int P,
                                  int inverse, const void* in, void* out, cudaStream_t stream) {
  cudaError_t err;
  if (tma_layout_permute(esize, B, N, H, d, layout, P, inverse, in, out, stream, &err)) return err;
  PermuteMap m;
  m.lay = make_layout(layout, N, P);
  m.N = N;
  m.row_bytes = (int64_t)H * d * esize;
  m.inverse = inverse;
  return launch_gather(in, out, (int64_t)B * N, m.row_bytes, m, stream);
}

cudaError_t launch_seq_head_repack(int esize, int P, int64_t n_local, int H, int d,
                                   int head_to_seq, const void* in, void* out,
                                   cudaStream_t stream) {
  cudaError_t err;
  if (tma_seq_head_repack(esize, P, n_local, H, d, head_to_seq, in, out, stream, &err)) return err;
  RepackMap m;
  m.ntot = (int64_t)P * n_local;
  m.P = P;
  m.run_bytes = (int64_t)(H / P) * d * esize;
  m.head_to_seq = head_to_seq;
  return launch_gather(in, out, m.ntot * P, m.run_bytes, m, stream);
}

}  // namespace rm
