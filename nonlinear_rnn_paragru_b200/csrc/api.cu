// api.cu -- the C ABI (include/pararnn.h): argument checks, workspace layout,
// TMA descriptors and kernel launches.  Host code only; every step of the
// solve runs in the kernels.
#include <cudaTypedefs.h>
#include <stdint.h>

#include <algorithm>

#include "common.cuh"

namespace pararnn {
int launch_gru_fwd(const CUtensorMap& tmap, bool bf16, const FwdParams& p, int nctas,
                   cudaStream_t stream);
int gru_chunk_steps();
int gru_max_cluster(bool bf16);
int gru_row_cluster(int T);
int gru_row_box_steps();
int gru_row_channels();
int launch_gru_row(const CUtensorMap& map, const FwdParams& p, bool f32, cudaStream_t stream);
int gru_row_max_steps();
int gru_row_cta_steps();
int gru_queue_resident();
int launch_gru_queue(const CUtensorMap& map, const CUtensorMap& hmap, const FwdParams& f,
                     unsigned* counter,
                     unsigned* seg_done, cudaStream_t stream);
int launch_lstm_fwd(const CUtensorMap& tmap, bool bf16, const FwdParams& p, int nctas,
                    cudaStream_t stream);
int lstm_chunk_steps();
int lstm_max_cluster(bool bf16);
int lstm_row_cluster(int T);
int lstm_row_cta_steps();
int lstm_row_box_steps();
int lstm_row_channels();
int launch_lstm_row(const CUtensorMap& map, const FwdParams& p, cudaStream_t stream);
int launch_lstm_queue(const CUtensorMap& map, const CUtensorMap& cmap, const CUtensorMap& hmap,
                      const FwdParams& f, unsigned* counter,
                      unsigned* seg_done, cudaStream_t stream);
int lstm_queue_resident();
int lstm_queue_box_steps();
int adjoint_row_cluster(int T);
int adjoint_row_channels();
int adjoint_row_box_steps(int which);
size_t adjoint_row_part_bytes(int G, int B, int T, int D);
size_t adjoint_queue_bytes(int B, int T, int D);
int adjoint_queue_box_steps(int which);
int adjoint_queue_channels();
int adjoint_queue_resident();
size_t adjoint_queue_lstm_bytes(int B, int T, int D);
int adjoint_queue_lstm_resident();
int adjoint_queue_lstm_channels();
int launch_adjoint_queue_lstm(const CUtensorMap* maps, const float* a, const float* bias,
                              const float* c0, const float* h0, float* du, float* da,
                              float* dbias, float* dc0, float* dh0, int B, int T, int D,
                              int* status, void* ws, uint64_t timeout_ns, int withhold_item,
                              cudaStream_t stream);
int launch_adjoint_queue(const CUtensorMap* maps, const float* a, const float* bias,
                         const float* h0, float* du, float* da, float* dbias, float* dh0, int B,
                         int T, int D, int* status, void* ws, uint64_t timeout_ns,
                         int withhold_item, cudaStream_t stream);
int launch_adjoint_row(const CUtensorMap* maps, const float* a, const float* bias,
                       const float* h0, float* du, float* da, float* dbias, float* dh0, int B,
                       int T, int D, int* status, void* ws, uint64_t timeout_ns,
                       int withhold_rank, cudaStream_t stream);
int launch_adjoint_row_lstm(const CUtensorMap* maps, const float* a, const float* bias,
                            const float* c0, const float* h0, float* du, float* da,
                            float* dbias, float* dc0, float* dh0, int B, int T, int D,
                            int* status, void* ws, uint64_t timeout_ns, int withhold_rank,
                            cudaStream_t stream);
size_t unfused_ws_bytes(int cell, int B, int T, int D);
int dense_max_d(bool simt);
int tc_operand_map(CUtensorMap* map, const float* base, int K, int rows, int Z, long long zstride);
int launch_tc_gemm(const CUtensorMap& ma, const CUtensorMap& mb, float* C, int M, int N, int K,
                   int Z, int store_mode, int* err, cudaStream_t stream);
size_t dense_ws_bytes(int B, int T, int D);
int dense_gru_solve(bool bf16, bool simt, const void* u, const float* W, const float* bias,
                    const float* h0, float* h, int B, int T, int D, float tol, int max_iters,
                    pararnn_stats* stats, void* workspace, cudaStream_t stream);
int unfused_solve(int cell, bool bf16, const void* u, const float* a, const float* bias,
                  const float* c0, const float* h0, float* c, float* h, int B, int T, int D,
                  float tol, int max_iters, pararnn_stats* stats, void* workspace,
                  cudaStream_t stream);
int shard_eval(int cell, bool bf16, const void* u, const float* a, const float* bias,
               const float* c_bound, const float* h_bound, const float* c, const float* h, int B,
               int Ts, int D, float* agg, float* last, float* rmax, void* workspace,
               cudaStream_t stream);
int shard_combine(int cell, const float* aggs, const float* lasts, int r, int B, int D,
                  float* din, float* bound, cudaStream_t stream);
int shard_apply(int cell, const float* din, float* c, float* h, int B, int Ts, int D,
                void* workspace, cudaStream_t stream);
int launch_decode_step(int cell, bool bf16, const void* u, const float* a, const float* bias,
                       const float* c_prev, const float* h_prev, float* c_next, float* h_next,
                       int B, int D, cudaStream_t stream);
int launch_seq_baseline(int cell, bool bf16, const void* u, const float* a, const float* bias,
                        const float* c0, const float* h0, float* c, float* h, int B, int T,
                        int D, cudaStream_t stream);
struct AdjParams;
int adjoint_chunk_steps(int cell);
size_t adjoint_ws_bytes(int cell, int B, int T, int D);
int launch_adjoint(int cell, bool bf16, const CUtensorMap* maps, const void* u, const float* a,
                   const float* bias, const float* c0, const float* h0, const float* c,
                   const float* h, const float* dLdh, float* du, float* da, float* dbias,
                   float* dc0, float* dh0, int B, int T, int D, int* status, void* ws,
                   uint64_t timeout_ns, int inject_chunk, cudaStream_t stream);
}  // namespace pararnn

using namespace pararnn;

namespace {

constexpr int kDefaultMaxIters = 64;
constexpr float kDefaultTol = 1e-6f;
constexpr unsigned kDefaultTimeoutUs = 2000000u;
constexpr int kMaxItersLimit = 1 << 16;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }

int resolve_max_iters(int m) { return m <= 0 ? kDefaultMaxIters : m; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// Tensor map over u [B][T][G][D] with a box of `ch` channels x G gates x tc steps.
int make_u_map(CUtensorMap* map, const void* u, bool bf16, int B, int T, int G, int D, int tc,
               int ch = kChan) {
  auto fn = encode_fn();
  if (fn == nullptr) return PARARNN_ERR_CUDA;
  const cuuint64_t es = bf16 ? 2 : 4;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)G, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {D * es, (cuuint64_t)G * D * es, (cuuint64_t)T * G * D * es};
  cuuint32_t box[4] = {(cuuint32_t)ch, (cuuint32_t)G, (cuuint32_t)tc, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                  const_cast<void*>(u), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PARARNN_OK : PARARNN_ERR_CUDA;
}

// Tensor map over an fp32 [B][T][D] array with a box of `ch` channels x tc steps.
int make_s_map(CUtensorMap* map, const float* x, int B, int T, int D, int tc, int ch = kChan) {
  auto fn = encode_fn();
  if (fn == nullptr) return PARARNN_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)T * D * 4};
  cuuint32_t box[3] = {(cuuint32_t)ch, (cuuint32_t)tc, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(x), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PARARNN_OK : PARARNN_ERR_CUDA;
}

int check_sizes(int B, int T, int D) {
  if (B < 1 || T < 1 || D < 1 || (D % 8) != 0) return PARARNN_ERR_INVALID_ARG;
  if ((long long)B * T * D > (1LL << 40)) return PARARNN_ERR_TOO_LARGE;
  return PARARNN_OK;
}

int rec_floats(int cell) { return cell == PARARNN_GRU ? 4 : 12; }

int chunk_steps(int cell) { return cell == PARARNN_GRU ? gru_chunk_steps() : lstm_chunk_steps(); }

// Records are kept per cluster chunk; the workspace is sized for clusters of
// at least kMinCluster CTAs (the launch checks the size it actually needs).
constexpr int kMinCluster = 8;

long long cluster_chunks(int cell, int B, int T, int D, int CL) {
  const int nC = cdiv(T, chunk_steps(cell));
  const int cl = std::min(nC, CL);
  return (long long)B * cdiv(D, kChan) * cdiv(nC, cl);
}

size_t fwd_ws(int cell, int B, int T, int D, int max_iters) {
  return fwd_ws_layout((size_t)cluster_chunks(cell, B, T, D, kMinCluster), max_iters,
                       rec_floats(cell), (size_t)B * D)
      .total;
}

// Largest usable cluster size for a cell's kernel on the current device.
int max_cluster(int cell, bool bf16) {
  static int cache[2][2][64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int& c = cache[cell][bf16 ? 1 : 0][dev];
  if (c == 0) c = cell == PARARNN_GRU ? gru_max_cluster(bf16) : lstm_max_cluster(bf16);
  return c;
}

// New epoch, ticket counter and stats; the per-channel indices and the
// histogram zeroed; and, for the look-back solve, its record flags cleared so
// that nothing another call left in the workspace can pass for a record.
// (`flags` is the segment-queue solve's per-tile segment counts when that
// solve runs.)
__global__ void fwd_init_kernel(WsHeader* hdr, pararnn_stats* stats, int* chan_k, size_t nch,
                                int* hist, int nhist, unsigned* flags, size_t nflags) {
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    unsigned e = (hdr->epoch + 1u) & 0x1fffffffu;
    if (e == 0u) e = 1u;
    hdr->epoch = e;
    hdr->ticket = 0u;
    stats->iters = 0;
    stats->max_residual = 0.f;
    stats->status = 0;
    stats->evals = 0;
  }
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const size_t i0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (chan_k)
    for (size_t i = i0; i < nch; i += stride) chan_k[i] = 0;
  if (hist)
    for (size_t i = i0; i < (size_t)nhist; i += stride) hist[i] = 0;
  for (size_t i = i0; i < nflags; i += stride) flags[i] = 0u;
}

__global__ void hist_kernel(const int* __restrict__ chan_k, size_t n, int* hist, int max_iters) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int k = chan_k[i];
  if (k > max_iters) k = max_iters + 1;  // never below tol within the cap
  atomicAdd(&hist[k], 1);
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? PARARNN_OK : PARARNN_ERR_CUDA; }

// between the segments of a long sequence: the row kernel's tile counter

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaGetLastError();
  return sms;
}

int forward(int cell, const void* u, int u_dtype, const float* a, const float* bias,
            const float* c0, const float* h0, float* c, float* h, int B, int T, int D,
            const pararnn_opts* opts, pararnn_stats* stats, int* iter_hist, void* workspace,
            size_t ws_bytes, cudaStream_t stream) {
  int rc = check_sizes(B, T, D);
  if (rc) return rc;
  if (u_dtype != PARARNN_F32 && u_dtype != PARARNN_BF16) return PARARNN_ERR_UNSUPPORTED_DTYPE;
  if (!u || !a || !h || !stats || !workspace) return PARARNN_ERR_INVALID_ARG;
  if (cell == PARARNN_LSTM && !c) return PARARNN_ERR_INVALID_ARG;
  if (!aligned(u, 16) || !aligned(h, 16) || (c && !aligned(c, 16)) || !aligned(a, 4) ||
      (bias && !aligned(bias, 4)) || (h0 && !aligned(h0, 4)) || (c0 && !aligned(c0, 4)) ||
      !aligned(stats, 4) || !aligned(workspace, 256) || (iter_hist && !aligned(iter_hist, 4)))
    return PARARNN_ERR_MISALIGNED;
  int* const chan_iters = opts ? opts->chan_iters : nullptr;
  if (chan_iters && !aligned(chan_iters, 4)) return PARARNN_ERR_MISALIGNED;
  const float tol = (opts && opts->tol > 0.f) ? opts->tol : kDefaultTol;
  const int max_iters = resolve_max_iters(opts ? opts->max_iters : 0);
  if (max_iters > kMaxItersLimit) return PARARNN_ERR_INVALID_ARG;
  const int G = cell == PARARNN_GRU ? 3 : 4;
  const int tc = chunk_steps(cell);
  const int nDT = cdiv(D, kChan), nC = cdiv(T, tc);
  int clmax = max_cluster(cell, u_dtype == PARARNN_BF16);
  if (clmax <= 0) return PARARNN_ERR_CUDA;
  if (opts && opts->max_cluster > 0) clmax = std::min(clmax, opts->max_cluster);
  const int CL = std::min(nC, clmax);
  const int nCC = cdiv(nC, CL);
  const long long nctas = (long long)B * nDT * nCC * CL;
  if (nctas >= (1LL << 31)) return PARARNN_ERR_TOO_LARGE;
  const long long ncc = (long long)B * nDT * nCC;
  const FwdWsLayout L = fwd_ws_layout((size_t)ncc, max_iters, rec_floats(cell), (size_t)B * D);
  if (ws_bytes < L.total) return PARARNN_ERR_WORKSPACE_TOO_SMALL;

  CUtensorMap map;
  rc = make_u_map(&map, u, u_dtype == PARARNN_BF16, B, T, G, D, tc);
  if (rc) return rc;

  unsigned char* ws = static_cast<unsigned char*>(workspace);
  FwdParams p;
  p.a = a;
  p.bias = bias;
  p.h0 = h0;
  p.c0 = c0;
  p.h = h;
  p.c = c;
  p.B = B;
  p.T = T;
  p.D = D;
  p.nDT = nDT;
  p.nC = nC;
  p.CL = CL;
  p.nCC = nCC;
  p.max_iters = max_iters;
  p.tol = tol;
  p.flags = opts ? opts->flags : 0u;
  p.apx_tau = (p.flags & PARARNN_FLAG_EXACT_STEPS) ? 0.f : kApxTau;
  // the row kernels' certifying check: ParaLSTM certifies below tol / 2 (a
  // margin for the fp32 rounding of a cell state that is not bounded)
  p.chk_tol = cell == PARARNN_LSTM ? 0.5f * tol : tol;
  p.spec_tau = tol > 0.f ? std::sqrt(p.chk_tol) : -1.f;
  p.inject_chunk = opts ? opts->inject_chunk : -1;
  p.timeout_ns = 1000ull * ((opts && opts->timeout_us) ? opts->timeout_us : kDefaultTimeoutUs);
  p.hdr = reinterpret_cast<WsHeader*>(ws);
  p.rec_flags = reinterpret_cast<unsigned*>(ws + L.flags);
  p.rec_vals = reinterpret_cast<float*>(ws + L.vals);
  p.chan_k = chan_iters ? chan_iters
                        : (iter_hist ? reinterpret_cast<int*>(ws + L.chan_k) : nullptr);
  p.stats = stats;
  p.u = u;
  p.t_base = 0;
  p.t_len = T;
  p.seg = 0;
  p.ld_h0 = D;
  p.seg_done = reinterpret_cast<unsigned*>(ws + L.seg);
  p.nitems = 0;
  p.withhold_item = (p.flags & PARARNN_FLAG_INJECT_WITHHOLD) ? p.inject_chunk : -1;

  // Row kernels: a cluster of CTAs per 8-channel tile holds a whole sequence
  // of up to 4096 steps (ParaGRU: bf16 or fp32 u; ParaLSTM: bf16 u).  Where a
  // smaller cluster of k CTAs already fills the SMs with the tiles (ParaGRU:
  // two CTAs per SM, 1024 steps per CTA; ParaLSTM: one, 512 steps), the
  // sequence is solved in segments of k CTAs' steps, in order, each segment
  // starting from the state the one before it converged to: the same work as
  // one solve over the whole sequence, with smaller clusters that fit the SMs
  // without gaps and shorter segments that converge in fewer iterations.  A
  // ParaGRU sequence longer than 4096 steps with at least one 8-channel tile
  // per SM is solved in 4096-step segments.  Otherwise, or on request, the
  // chunked cluster + look-back solve.
  const bool force = opts && (opts->flags & PARARNN_FLAG_FORCE_CHUNKED);
  const bool bf16 = u_dtype == PARARNN_BF16;
  const long long tiles8 = (long long)B * ((D + 7) / 8);
  const bool row_gru = cell == PARARNN_GRU && !force &&
                       (gru_row_cluster(T) > 0 || tiles8 >= sm_count());
  const bool row_lstm = cell == PARARNN_LSTM && bf16 && lstm_row_cluster(T) > 0 && !force;
  // ParaGRU with bf16 u and at least one 8-channel tile per resident CTA of
  // the segment-queue solve: all segments of all tiles in one launch
  const bool force_row = opts && (opts->flags & PARARNN_FLAG_FORCE_ROW);
  const bool queue_gru = row_gru && bf16 && !force_row &&
                         tiles8 >= (long long)std::max(1, gru_queue_resident());
  // ParaLSTM (bf16 u, any T) with at least one 8-channel tile per resident CTA
  // of the segment-queue solve (four per SM): every 128-step segment in one
  // launch
  const bool queue_lstm = cell == PARARNN_LSTM && bf16 && !force && !force_row &&
                          tiles8 >= (long long)std::max(1, lstm_queue_resident());
  const size_t nch = (size_t)B * D;
  const int nhist = max_iters + 2;
  unsigned* const seg_done = p.seg_done;
  const size_t nflags = (queue_gru || queue_lstm) ? (size_t)tiles8
                                  : ((row_gru || row_lstm) ? 0 : (size_t)ncc * (size_t)(max_iters + 1));
  const size_t ninit = std::max(p.chan_k ? nch : (size_t)1, nflags);
  const unsigned igrid = (unsigned)std::min<size_t>((ninit + 255) / 256, 1024);
  fwd_init_kernel<<<igrid, 256, 0, stream>>>(p.hdr, stats, p.chan_k, nch, iter_hist, nhist,
                                             (queue_gru || queue_lstm) ? seg_done : p.rec_flags,
                                             nflags);
  if (cudaGetLastError() != cudaSuccess) return PARARNN_ERR_CUDA;
  int e = 0;
  if (queue_gru) {
    CUtensorMap rmap;
    rc = make_u_map(&rmap, u, true, B, T, G, D, gru_row_box_steps(), gru_row_channels());
    CUtensorMap hmap;  // the states, stored by the same 256-step boxes
    if (!rc) rc = make_s_map(&hmap, h, B, T, D, gru_row_box_steps(), gru_row_channels());
    if (rc) return rc;
    e = launch_gru_queue(rmap, hmap, p, &p.hdr->ticket, seg_done, stream);
  } else if (queue_lstm) {
    CUtensorMap rmap;
    rc = make_u_map(&rmap, u, true, B, T, G, D, lstm_queue_box_steps(), lstm_row_channels());
    CUtensorMap cmap, hmap;  // the states, stored by the same 128-step boxes
    if (!rc) rc = make_s_map(&cmap, c, B, T, D, lstm_queue_box_steps(), lstm_row_channels());
    if (!rc) rc = make_s_map(&hmap, h, B, T, D, lstm_queue_box_steps(), lstm_row_channels());
    if (rc) return rc;
    e = launch_lstm_queue(rmap, cmap, hmap, p, &p.hdr->ticket, seg_done, stream);
  } else if (row_gru) {
    CUtensorMap rmap;
    rc = make_u_map(&rmap, u, bf16, B, T, G, D, gru_row_box_steps(), gru_row_channels());
    if (rc) return rc;
    int seg = gru_row_max_steps();
    if (T <= seg) {
      seg = T;
      for (int k = 1; k < gru_row_cluster(T); k *= 2)
        if (k * tiles8 >= 2 * sm_count()) {  // two CTAs per SM
          seg = k * gru_row_cta_steps();
          break;
        }
    }
    for (int s0 = 0; s0 < T && e == 0; s0 += seg) {
      FwdParams ps = p;
      ps.t_base = s0;
      ps.t_len = std::min(seg, T - s0);
      ps.seg = s0 / seg;
      if (s0 > 0) {
        ps.h0 = h + (size_t)(s0 - 1) * D;  // the last state of the segment before
        ps.ld_h0 = (long long)T * D;
      }
      e = launch_gru_row(rmap, ps, !bf16, stream);
    }
  } else if (row_lstm) {
    CUtensorMap rmap;
    rc = make_u_map(&rmap, u, true, B, T, G, D, lstm_row_box_steps(), lstm_row_channels());
    if (rc) return rc;
    int seg = T;
    for (int k = 1; k < lstm_row_cluster(T); k *= 2)
      if (k * tiles8 >= sm_count()) {
        seg = k * lstm_row_cta_steps();
        break;
      }
    for (int s0 = 0; s0 < T && e == 0; s0 += seg) {
      FwdParams ps = p;
      ps.t_base = s0;
      ps.t_len = std::min(seg, T - s0);
      if (s0 > 0) {  // the last (c, h) of the segment before
        ps.c0 = c + (size_t)(s0 - 1) * D;
        ps.h0 = h + (size_t)(s0 - 1) * D;
        ps.ld_h0 = (long long)T * D;
      }
      e = launch_lstm_row(rmap, ps, stream);
    }
  } else {
    e = cell == PARARNN_GRU ? launch_gru_fwd(map, bf16, p, (int)nctas, stream)
                            : launch_lstm_fwd(map, bf16, p, (int)nctas, stream);
  }
  if (e != 0) return PARARNN_ERR_CUDA;
  if (iter_hist) {
    hist_kernel<<<(unsigned)((nch + 255) / 256), 256, 0, stream>>>(p.chan_k, nch, iter_hist,
                                                                     max_iters);
    if (cudaGetLastError() != cudaSuccess) return PARARNN_ERR_CUDA;
  }
  return PARARNN_OK;
}

}  // namespace

extern "C" {

size_t pararnn_workspace_size(int cell, int B, int T, int D, int max_iters, int adjoint) {
  if (cell != PARARNN_GRU && cell != PARARNN_LSTM) return 0;
  if (check_sizes(B, T, D) != PARARNN_OK) return 0;
  if (adjoint) return adjoint_ws_bytes(cell, B, T, D);
  const int m = resolve_max_iters(max_iters);
  if (m > kMaxItersLimit) return 0;
  return fwd_ws(cell, B, T, D, m);
}

int pararnn_workspace_init(void* workspace, size_t ws_bytes, pararnn_stream_t stream) {
  if (!workspace) return PARARNN_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(workspace, 0, ws_bytes, (cudaStream_t)stream));
}

int pararnn_gru_solve(const void* u, int u_dtype, const float* a, const float* bias,
                      const float* h0, float* h, int B, int T, int D, const pararnn_opts* opts,
                      pararnn_stats* stats, int* iter_hist, void* workspace, size_t ws_bytes,
                      pararnn_stream_t stream) {
  return forward(PARARNN_GRU, u, u_dtype, a, bias, nullptr, h0, nullptr, h, B, T, D, opts, stats,
                 iter_hist, workspace, ws_bytes, (cudaStream_t)stream);
}

int pararnn_lstm_solve(const void* u, int u_dtype, const float* a, const float* bias,
                       const float* c0, const float* h0, float* c, float* h, int B, int T, int D,
                       const pararnn_opts* opts, pararnn_stats* stats, int* iter_hist,
                       void* workspace, size_t ws_bytes, pararnn_stream_t stream) {
  return forward(PARARNN_LSTM, u, u_dtype, a, bias, c0, h0, c, h, B, T, D, opts, stats, iter_hist,
                 workspace, ws_bytes, (cudaStream_t)stream);
}

int pararnn_adjoint(int cell, const void* u, int u_dtype, const float* a, const float* bias,
                    const float* c0, const float* h0, const float* c, const float* h,
                    const float* dLdh, float* du, float* da, float* dbias, float* dc0, float* dh0,
                    int B, int T, int D, int* status, void* workspace, size_t ws_bytes,
                    pararnn_stream_t stream) {
  return pararnn_adjoint_ex(cell, u, u_dtype, a, bias, c0, h0, c, h, dLdh, du, da, dbias, dc0,
                            dh0, B, T, D, status, workspace, ws_bytes, nullptr, stream);
}

int pararnn_adjoint_ex(int cell, const void* u, int u_dtype, const float* a, const float* bias,
                       const float* c0, const float* h0, const float* c, const float* h,
                       const float* dLdh, float* du, float* da, float* dbias, float* dc0,
                       float* dh0, int B, int T, int D, int* status, void* workspace,
                       size_t ws_bytes, const pararnn_opts* opts, pararnn_stream_t stream) {
  const uint64_t timeout_ns =
      1000ull * ((opts && opts->timeout_us) ? opts->timeout_us : kDefaultTimeoutUs);
  const bool inject = opts && (opts->flags & PARARNN_FLAG_INJECT_WITHHOLD);
  const int inject_chunk = inject ? opts->inject_chunk : -1;
  if (cell != PARARNN_GRU && cell != PARARNN_LSTM) return PARARNN_ERR_INVALID_ARG;
  int rc = check_sizes(B, T, D);
  if (rc) return rc;
  if (u_dtype != PARARNN_F32 && u_dtype != PARARNN_BF16) return PARARNN_ERR_UNSUPPORTED_DTYPE;
  if (!u || !a || !h || !dLdh || !du || !da || !status || !workspace)
    return PARARNN_ERR_INVALID_ARG;
  if (cell == PARARNN_LSTM && !c) return PARARNN_ERR_INVALID_ARG;
  if (cell == PARARNN_GRU && (c || c0 || dc0)) return PARARNN_ERR_INVALID_ARG;
  if (!aligned(u, 16) || !aligned(h, 16) || !aligned(dLdh, 16) || !aligned(du, 16) ||
      (c && !aligned(c, 16)) || !aligned(a, 4) || !aligned(da, 4) || (bias && !aligned(bias, 4)) ||
      (dbias && !aligned(dbias, 4)) || (h0 && !aligned(h0, 4)) || (c0 && !aligned(c0, 4)) ||
      (dh0 && !aligned(dh0, 4)) || (dc0 && !aligned(dc0, 4)) || !aligned(status, 4) ||
      !aligned(workspace, 256))
    return PARARNN_ERR_MISALIGNED;
  if (ws_bytes < adjoint_ws_bytes(cell, B, T, D)) return PARARNN_ERR_WORKSPACE_TOO_SMALL;
  const int G = cell == PARARNN_GRU ? 3 : 4;
  const bool force_row = opts && (opts->flags & PARARNN_FLAG_FORCE_ROW);
  // the queue and whole-sequence kernels stage each tile's rows of a, bias,
  // h0 (c0) with 1-D bulk copies, which take 16-byte aligned addresses only
  const bool rows16 = aligned(a, 16) && (!bias || aligned(bias, 16)) &&
                      (!h0 || aligned(h0, 16)) && (!c0 || aligned(c0, 16));
  // ParaGRU, bf16 projections, at least one 32-channel tile per resident CTA
  // of the queue adjoint: every 128-step segment in one launch, last first
  if (cell == PARARNN_GRU && u_dtype == PARARNN_BF16 && !force_row && rows16 &&
      (long long)B * ((D + 31) / 32) >= (long long)std::max(1, adjoint_queue_resident()) &&
      kWsHeaderBytes + adjoint_queue_bytes(B, T, D) <= ws_bytes) {
    const int ch = adjoint_queue_channels();
    CUtensorMap qmaps[3];  // u, h (states before each step), dL/dh
    rc = make_u_map(&qmaps[0], u, true, B, T, G, D, adjoint_queue_box_steps(0), ch);
    if (!rc) rc = make_s_map(&qmaps[1], h, B, T, D, adjoint_queue_box_steps(1), ch);
    if (!rc) rc = make_s_map(&qmaps[2], dLdh, B, T, D, adjoint_queue_box_steps(2), ch);
    if (rc) return rc;
    const int e = launch_adjoint_queue(qmaps, a, bias, h0, du, da, dbias, dh0, B, T, D, status,
                                       static_cast<unsigned char*>(workspace) + kWsHeaderBytes,
                                       timeout_ns, inject_chunk, (cudaStream_t)stream);
    return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
  }
  // ParaLSTM likewise (32-channel tiles, one 16-warp CTA per SM)
  if (cell == PARARNN_LSTM && u_dtype == PARARNN_BF16 && !force_row && rows16 &&
      (long long)B * ((D + 31) / 32) >= (long long)std::max(1, adjoint_queue_lstm_resident()) &&
      kWsHeaderBytes + adjoint_queue_lstm_bytes(B, T, D) <= ws_bytes) {
    const int ch = adjoint_queue_lstm_channels();
    const int tc = adjoint_queue_box_steps(0);
    CUtensorMap qmaps[4];  // u, c and h (states before each step), dL/dh
    rc = make_u_map(&qmaps[0], u, true, B, T, G, D, tc, ch);
    if (!rc) rc = make_s_map(&qmaps[1], c, B, T, D, tc, ch);
    if (!rc) rc = make_s_map(&qmaps[2], h, B, T, D, tc, ch);
    if (!rc) rc = make_s_map(&qmaps[3], dLdh, B, T, D, tc, ch);
    if (rc) return rc;
    const int e = launch_adjoint_queue_lstm(
        qmaps, a, bias, c0, h0, du, da, dbias, dc0, dh0, B, T, D, status,
        static_cast<unsigned char*>(workspace) + kWsHeaderBytes, timeout_ns, inject_chunk,
        (cudaStream_t)stream);
    return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
  }
  // bf16 projections, sequences of up to 4096 steps: a cluster of CTAs per
  // 8-channel tile holds the whole sequence (no look-back)
  if (u_dtype == PARARNN_BF16 && rows16 && adjoint_row_cluster(T) > 0 &&
      kWsHeaderBytes + adjoint_row_part_bytes(G, B, T, D) <= ws_bytes) {
    const int ch = adjoint_row_channels();
    CUtensorMap rmaps[4];
    int e;
    if (cell == PARARNN_GRU) {  // u, h (states before each step), dL/dh
      rc = make_u_map(&rmaps[0], u, true, B, T, G, D, adjoint_row_box_steps(0), ch);
      if (!rc) rc = make_s_map(&rmaps[1], h, B, T, D, adjoint_row_box_steps(1), ch);
      if (!rc) rc = make_s_map(&rmaps[2], dLdh, B, T, D, adjoint_row_box_steps(2), ch);
      if (rc) return rc;
      e = launch_adjoint_row(rmaps, a, bias, h0, du, da, dbias, dh0, B, T, D, status, workspace,
                             timeout_ns, inject_chunk, (cudaStream_t)stream);
    } else {  // u, c and h (states before each step), dL/dh
      rc = make_u_map(&rmaps[0], u, true, B, T, G, D, adjoint_row_box_steps(0), ch);
      if (!rc) rc = make_s_map(&rmaps[1], c, B, T, D, adjoint_row_box_steps(1), ch);
      if (!rc) rc = make_s_map(&rmaps[2], h, B, T, D, adjoint_row_box_steps(1), ch);
      if (!rc) rc = make_s_map(&rmaps[3], dLdh, B, T, D, adjoint_row_box_steps(2), ch);
      if (rc) return rc;
      e = launch_adjoint_row_lstm(rmaps, a, bias, c0, h0, du, da, dbias, dc0, dh0, B, T, D,
                                  status, workspace, timeout_ns, inject_chunk,
                                  (cudaStream_t)stream);
    }
    return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
  }
  const int tc = adjoint_chunk_steps(cell);
  CUtensorMap maps[4];  // u, h, c (ParaLSTM; h again for ParaGRU), dL/dh
  rc = make_u_map(&maps[0], u, u_dtype == PARARNN_BF16, B, T, G, D, tc);
  if (!rc) rc = make_s_map(&maps[1], h, B, T, D, tc);
  if (!rc) rc = make_s_map(&maps[2], c ? c : h, B, T, D, tc);
  if (!rc) rc = make_s_map(&maps[3], dLdh, B, T, D, tc);
  if (rc) return rc;
  const int e = launch_adjoint(cell, u_dtype == PARARNN_BF16, maps, u, a, bias, c0, h0, c, h, dLdh,
                               du, da, dbias, dc0, dh0, B, T, D, status, workspace,
                               timeout_ns, inject_chunk, (cudaStream_t)stream);
  return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
}

int pararnn_seq_baseline(int cell, const void* u, int u_dtype, const float* a, const float* bias,
                         const float* c0, const float* h0, float* c, float* h, int B, int T, int D,
                         pararnn_stream_t stream) {
  if (cell != PARARNN_GRU && cell != PARARNN_LSTM) return PARARNN_ERR_INVALID_ARG;
  int rc = check_sizes(B, T, D);
  if (rc) return rc;
  if (u_dtype != PARARNN_F32 && u_dtype != PARARNN_BF16) return PARARNN_ERR_UNSUPPORTED_DTYPE;
  if (!u || !a || !h || (cell == PARARNN_LSTM && !c)) return PARARNN_ERR_INVALID_ARG;
  if (cell == PARARNN_GRU && (c || c0)) return PARARNN_ERR_INVALID_ARG;
  const int e = launch_seq_baseline(cell, u_dtype == PARARNN_BF16, u, a, bias, c0, h0, c, h, B, T,
                                    D, (cudaStream_t)stream);
  return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
}

size_t pararnn_shard_workspace_size(int cell, int B, int Ts, int D) {
  if (cell != PARARNN_GRU && cell != PARARNN_LSTM) return 0;
  if (check_sizes(B, Ts, D)) return 0;
  return unfused_ws_bytes(cell, B, Ts, D);
}

int pararnn_shard_eval(int cell, const void* u, int u_dtype, const float* a, const float* bias,
                       const float* c_bound, const float* h_bound, const float* c,
                       const float* h, int B, int Ts, int D, float* agg, float* last,
                       float* rmax, void* workspace, size_t ws_bytes, pararnn_stream_t stream) {
  if (cell != PARARNN_GRU && cell != PARARNN_LSTM) return PARARNN_ERR_INVALID_ARG;
  int rc = check_sizes(B, Ts, D);
  if (rc) return rc;
  if (u_dtype != PARARNN_F32 && u_dtype != PARARNN_BF16) return PARARNN_ERR_UNSUPPORTED_DTYPE;
  const bool lstm = cell == PARARNN_LSTM;
  if (!u || !a || !h || !agg || !last || !rmax || !workspace || (lstm && !c))
    return PARARNN_ERR_INVALID_ARG;
  if (!lstm && (c || c_bound)) return PARARNN_ERR_INVALID_ARG;
  if (!aligned(u, u_dtype == PARARNN_BF16 ? 2 : 4) || !aligned(a, 4) ||
      (bias && !aligned(bias, 4)) || (c_bound && !aligned(c_bound, 4)) ||
      (h_bound && !aligned(h_bound, 4)) || (c && !aligned(c, 4)) || !aligned(h, 4) ||
      !aligned(agg, 4) || !aligned(last, 4) || !aligned(rmax, 4) || !aligned(workspace, 256))
    return PARARNN_ERR_MISALIGNED;
  if (ws_bytes < unfused_ws_bytes(cell, B, Ts, D)) return PARARNN_ERR_WORKSPACE_TOO_SMALL;
  const int e = shard_eval(cell, u_dtype == PARARNN_BF16, u, a, bias, c_bound, h_bound, c, h, B,
                           Ts, D, agg, last, rmax, workspace, (cudaStream_t)stream);
  return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
}

int pararnn_shard_combine(int cell, const float* aggs, const float* lasts, int W, int r, int B,
                          int D, float* din, float* bound, pararnn_stream_t stream) {
  if (cell != PARARNN_GRU && cell != PARARNN_LSTM) return PARARNN_ERR_INVALID_ARG;
  if (W < 1 || r < 0 || r >= W || B < 1 || D < 1) return PARARNN_ERR_INVALID_ARG;
  if (!aggs || !lasts || !din || (r > 0 && !bound)) return PARARNN_ERR_INVALID_ARG;
  if (!aligned(aggs, 4) || !aligned(lasts, 4) || !aligned(din, 4) || (bound && !aligned(bound, 4)))
    return PARARNN_ERR_MISALIGNED;
  const int e = shard_combine(cell, aggs, lasts, r, B, D, din, bound, (cudaStream_t)stream);
  return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
}

int pararnn_shard_apply(int cell, const float* din, float* c, float* h, int B, int Ts, int D,
                        void* workspace, size_t ws_bytes, pararnn_stream_t stream) {
  if (cell != PARARNN_GRU && cell != PARARNN_LSTM) return PARARNN_ERR_INVALID_ARG;
  int rc = check_sizes(B, Ts, D);
  if (rc) return rc;
  const bool lstm = cell == PARARNN_LSTM;
  if (!din || !h || !workspace || (lstm && !c) || (!lstm && c)) return PARARNN_ERR_INVALID_ARG;
  if (!aligned(din, 4) || !aligned(h, 4) || (c && !aligned(c, 4)) || !aligned(workspace, 256))
    return PARARNN_ERR_MISALIGNED;
  if (ws_bytes < unfused_ws_bytes(cell, B, Ts, D)) return PARARNN_ERR_WORKSPACE_TOO_SMALL;
  const int e = shard_apply(cell, din, c, h, B, Ts, D, workspace, (cudaStream_t)stream);
  return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
}

size_t pararnn_unfused_workspace_size(int cell, int B, int T, int D) {
  if (cell != PARARNN_GRU && cell != PARARNN_LSTM) return 0;
  if (check_sizes(B, T, D)) return 0;
  return unfused_ws_bytes(cell, B, T, D);
}

int pararnn_solve_unfused(int cell, const void* u, int u_dtype, const float* a, const float* bias,
                          const float* c0, const float* h0, float* c, float* h, int B, int T,
                          int D, const pararnn_opts* opts, pararnn_stats* stats, void* workspace,
                          size_t ws_bytes, pararnn_stream_t stream) {
  if (cell != PARARNN_GRU && cell != PARARNN_LSTM) return PARARNN_ERR_INVALID_ARG;
  int rc = check_sizes(B, T, D);
  if (rc) return rc;
  if (u_dtype != PARARNN_F32 && u_dtype != PARARNN_BF16) return PARARNN_ERR_UNSUPPORTED_DTYPE;
  if (!u || !a || !h || !stats || !workspace) return PARARNN_ERR_INVALID_ARG;
  if (cell == PARARNN_LSTM && !c) return PARARNN_ERR_INVALID_ARG;
  if (cell == PARARNN_GRU && (c || c0)) return PARARNN_ERR_INVALID_ARG;
  if (!aligned(u, u_dtype == PARARNN_BF16 ? 2 : 4) || !aligned(h, 4) || (c && !aligned(c, 4)) ||
      !aligned(a, 4) || (bias && !aligned(bias, 4)) || (h0 && !aligned(h0, 4)) ||
      (c0 && !aligned(c0, 4)) || !aligned(stats, 4) || !aligned(workspace, 256))
    return PARARNN_ERR_MISALIGNED;
  if (ws_bytes < unfused_ws_bytes(cell, B, T, D)) return PARARNN_ERR_WORKSPACE_TOO_SMALL;
  const float tol = (opts && opts->tol > 0.f) ? opts->tol : kDefaultTol;
  const int max_iters = resolve_max_iters(opts ? opts->max_iters : 0);
  if (max_iters > kMaxItersLimit) return PARARNN_ERR_INVALID_ARG;
  const int e = unfused_solve(cell, u_dtype == PARARNN_BF16, u, a, bias, c0, h0, c, h, B, T, D,
                              tol, max_iters, stats, workspace, (cudaStream_t)stream);
  return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
}

int pararnn_dense_matmul(const float* A, const float* Bm, float* C, int M, int N, int K, int Z,
                         int store_mode, int* err, pararnn_stream_t stream) {
  if (!A || !Bm || !C || !err || M < 1 || N < 1 || K < 1 || Z < 1 || (K % 4) != 0 ||
      store_mode < 0 || store_mode > 3)
    return PARARNN_ERR_INVALID_ARG;
  if ((long long)M * N * Z >= (1LL << 40) || M >= (1 << 30) || N >= (1 << 30))
    return PARARNN_ERR_TOO_LARGE;
  if (!aligned(A, 16) || !aligned(Bm, 16) || !aligned(C, 16) || !aligned(err, 4))
    return PARARNN_ERR_MISALIGNED;
  CUtensorMap ma, mb;
  if (tc_operand_map(&ma, A, K, M, Z, (long long)M * K) ||
      tc_operand_map(&mb, Bm, K, N, Z, (long long)N * K))
    return PARARNN_ERR_CUDA;
  const int e = launch_tc_gemm(ma, mb, C, M, N, K, Z, store_mode, err, (cudaStream_t)stream);
  return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
}

size_t pararnn_dense_workspace_size(int B, int T, int D) {
  if (check_sizes(B, T, D) || D > dense_max_d(false)) return 0;
  return dense_ws_bytes(B, T, D);
}

int pararnn_dense_gru_solve(const void* u, int u_dtype, const float* W, const float* bias,
                            const float* h0, float* h, int B, int T, int D,
                            const pararnn_opts* opts, pararnn_stats* stats, void* workspace,
                            size_t ws_bytes, pararnn_stream_t stream) {
  int rc = check_sizes(B, T, D);
  if (rc) return rc;
  const bool simt = opts && (opts->flags & PARARNN_FLAG_DENSE_SIMT);
  if (D > dense_max_d(simt)) return PARARNN_ERR_INVALID_ARG;
  if ((long long)B * T >= (1LL << 31)) return PARARNN_ERR_TOO_LARGE;
  if (u_dtype != PARARNN_F32 && u_dtype != PARARNN_BF16) return PARARNN_ERR_UNSUPPORTED_DTYPE;
  if (!u || !W || !h || !stats || !workspace) return PARARNN_ERR_INVALID_ARG;
  if (!aligned(u, u_dtype == PARARNN_BF16 ? 2 : 4) || !aligned(W, 16) || !aligned(h, 16) ||
      (bias && !aligned(bias, 4)) || (h0 && !aligned(h0, 16)) || !aligned(stats, 4) ||
      !aligned(workspace, 256))
    return PARARNN_ERR_MISALIGNED;
  if (ws_bytes < dense_ws_bytes(B, T, D)) return PARARNN_ERR_WORKSPACE_TOO_SMALL;
  const float tol = (opts && opts->tol > 0.f) ? opts->tol : kDefaultTol;
  const int max_iters = resolve_max_iters(opts ? opts->max_iters : 0);
  if (max_iters > kMaxItersLimit) return PARARNN_ERR_INVALID_ARG;
  const int e = dense_gru_solve(u_dtype == PARARNN_BF16, simt, u, W, bias, h0, h, B, T, D, tol,
                                max_iters, stats, workspace, (cudaStream_t)stream);
  return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
}

// Shared checks of the two single-step entry points.
static int step_args(const void* u_t, int u_dtype, const float* a, const float* bias, int B, int D) {
  const int rc = check_sizes(B, 1, D);
  if (rc) return rc;
  if (u_dtype != PARARNN_F32 && u_dtype != PARARNN_BF16) return PARARNN_ERR_UNSUPPORTED_DTYPE;
  if (!u_t || !a) return PARARNN_ERR_INVALID_ARG;
  if (!aligned(u_t, u_dtype == PARARNN_BF16 ? 2 : 4) || !aligned(a, 4) || (bias && !aligned(bias, 4)))
    return PARARNN_ERR_MISALIGNED;
  return PARARNN_OK;
}

int pararnn_gru_step(const void* u_t, int u_dtype, const float* a, const float* bias,
                     const float* h_prev, float* h_next, int B, int D, pararnn_stream_t stream) {
  int rc = step_args(u_t, u_dtype, a, bias, B, D);
  if (rc) return rc;
  if (!h_next) return PARARNN_ERR_INVALID_ARG;
  if ((h_prev && !aligned(h_prev, 4)) || !aligned(h_next, 4)) return PARARNN_ERR_MISALIGNED;
  const int e = launch_decode_step(PARARNN_GRU, u_dtype == PARARNN_BF16, u_t, a, bias, nullptr,
                                   h_prev, nullptr, h_next, B, D, (cudaStream_t)stream);
  return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
}

int pararnn_lstm_step(const void* u_t, int u_dtype, const float* a, const float* bias,
                      const float* c_prev, const float* h_prev, float* c_next, float* h_next,
                      int B, int D, pararnn_stream_t stream) {
  int rc = step_args(u_t, u_dtype, a, bias, B, D);
  if (rc) return rc;
  if (!c_next || !h_next || c_next == h_next) return PARARNN_ERR_INVALID_ARG;
  if ((c_prev && !aligned(c_prev, 4)) || (h_prev && !aligned(h_prev, 4)) ||
      !aligned(c_next, 4) || !aligned(h_next, 4))
    return PARARNN_ERR_MISALIGNED;
  const int e = launch_decode_step(PARARNN_LSTM, u_dtype == PARARNN_BF16, u_t, a, bias, c_prev,
                                   h_prev, c_next, h_next, B, D, (cudaStream_t)stream);
  return e == 0 ? PARARNN_OK : PARARNN_ERR_CUDA;
}

const char* pararnn_strerror(int code) {
  switch (code) {
    case PARARNN_OK: return "ok";
    case PARARNN_ERR_INVALID_ARG: return "invalid argument (null pointer, size or cell)";
    case PARARNN_ERR_UNSUPPORTED_DTYPE: return "unsupported dtype for u (want f32 or bf16)";
    case PARARNN_ERR_WORKSPACE_TOO_SMALL: return "workspace smaller than pararnn_workspace_size()";
    case PARARNN_ERR_CUDA: return "CUDA error while setting up or launching a kernel";
    case PARARNN_ERR_MISALIGNED: return "pointer misaligned (16 B for tensors, 4 B for vectors)";
    case PARARNN_ERR_TOO_LARGE: return "problem too large for the index types";
    default: return "unknown pararnn error code";
  }
}

}  // extern "C"
