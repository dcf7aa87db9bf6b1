// The QSA layer for one prefill whose inputs and output live in host memory: the copies in,
// the kernels and the copy out, scheduled on three streams so that transfers overlap compute.
//
// "Qwen3.8-Flash-Next architecture" (flozi.net), "Der Weg eines Tokens durch das Modell", item 2:
// the layer pools the indexer keys, selects each query's blocks and attends over them.  A prefill
// is causal, which lets the transfers start the work early:
//   * the pooling and selection of query rows [lo, hi) need only the indexer keys of the positions
//     before q_pos0 + hi and the indexer queries of those rows, so ki and qi are sent first, in
//     `sel_chunks` causal row chunks, and each chunk's pooling + selection starts when it has
//     arrived;
//   * the attention of rows [lo, hi) needs only their q and the K/V of the positions before
//     q_pos0 + hi, so q, k and v follow in `chunks` causal row chunks (K/V sent only up to each
//     chunk's end, never twice), each chunk's attention starts when it has arrived, and its output
//     goes back on a second copy stream while the next chunk is computed (PCIe is full duplex).
// Chunking needs one sequence (B = 1: a chunk's rows are contiguous in every tensor); the
// selection chunks also need a window that ends the context (Tk = q_pos0 + Tq) starting on a block
// boundary.  Otherwise the call sends everything first and runs each step once.  Chunk bounds are
// the same as the binding's: attention chunks on multiples of 16 rows (the query-tile attention
// groups rows 16 at a time from a call's first row, so the tiles, and the bits, are the same as in
// one call), selection chunks on multiples of 4.
//
// The steps are the library's own entry points (qsa_pool_block_keys_rope, qsa_rope_index_queries_rope,
// qsa_select_topk, and qsa_interleave_kv + qsa_sparse_attn_prefill_kv, or qsa_sparse_attn_prefill_ws);
// this file only moves data and orders streams.  With the automatic attention path and a shape the
// interleaved-K/V attention takes, each chunk interleaves only the K/V positions that arrived with
// it (the block that straddles the previous chunk's end is rewritten whole), so K and V are
// interleaved once per call, not once per chunk.  Copies are one cudaMemcpyAsync per contiguous range.
#include <algorithm>
#include <cmath>
#include <mutex>
#include <vector>

#include "launch.h"
#include "qsa.h"

namespace qsa {
namespace {

constexpr int kMaxDev = 64;
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Shape {
  int B, Tq, Tk, Hq, Hkv, D, Hi, Di, k, blk;
  long long q_pos0;
  bool rope;
  int chunks, sel_chunks;
};

// Row bounds of the attention chunks and of the selection chunks.  chunks == 0 (automatic, B = 1):
// three chunks of a quarter of the rows, then chunks that halve what is left down to about 2048
// rows.  The selection runs first, so the early chunks' inputs have arrived before they start
// even when they are large; large chunks leave fewer partial last waves of the attention's
// persistent CTAs, and the small last ones leave little output to copy back after the last kernel.
void chunk_bounds(const Shape& s, std::vector<int>& att, std::vector<int>& sel) {
  att.assign(1, 0);
  if (s.chunks == 0 && s.B == 1) {
    const long long T = s.Tq;
    auto push = [&](long long e) {
      e = e / 16 * 16;
      if (e > att.back() && e < T) att.push_back(static_cast<int>(e));
    };
    push(T / 4);
    push(T / 2);
    push(3 * T / 4);
    for (long long rem = T - 3 * T / 4; rem > 2048;) {
      rem /= 2;
      push(T - rem);
    }
  } else {
    const int n = s.B == 1 ? std::max(1, std::min(s.chunks, s.Tq)) : 1;
    for (int c = 1; c < n; ++c) att.push_back(static_cast<int>((static_cast<long long>(s.Tq) * c / n) / 16 * 16));
  }
  att.push_back(s.Tq);
  const bool can = s.B == 1 && s.q_pos0 % 4 == 0 && static_cast<long long>(s.Tk) == s.q_pos0 + s.Tq;
  const int ns = can ? std::max(1, std::min(s.sel_chunks, s.Tq / 4)) : 1;
  sel.assign(1, 0);
  for (int c = 1; c < ns; ++c) sel.push_back(static_cast<int>((static_cast<long long>(s.Tq) * c / ns) / 4 * 4));
  sel.push_back(s.Tq);
}

// Byte offsets of the regions of the device scratch buffer (each 256-byte aligned).
struct Layout {
  size_t q, k, v, qi, ki, kp, qr, out, idx, lse, sel_ws, att_ws, kv, total;
  size_t sel_ws_bytes, att_ws_bytes;
};

Layout layout(const Shape& s) {
  std::vector<int> att, sel;
  chunk_bounds(s, att, sel);
  const size_t B = s.B;
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes);
    return o;
  };
  L.q = take(B * s.Tq * s.Hq * s.D * 2);
  L.k = take(B * s.Tk * s.Hkv * s.D * 2);
  L.v = take(B * s.Tk * s.Hkv * s.D * 2);
  L.qi = take(B * s.Tq * s.Hi * s.Di * 2);
  L.ki = take(B * s.Tk * s.Di * 2);
  L.kp = take(B * (s.Tk / s.blk) * s.Di * 2);
  L.qr = s.rope ? take(B * s.Tq * s.Hi * s.Di * 2) : 0;
  L.out = take(B * s.Tq * s.Hq * s.D * 2);
  L.idx = take(B * s.Tq * static_cast<size_t>(s.k) * 4);
  L.lse = take(B * s.Tq * s.Hq * 4);
  size_t sws = 0;
  const int ns = static_cast<int>(sel.size()) - 1;
  for (int c = 0; c < ns; ++c) {
    const int rows = sel[c + 1] - sel[c];
    const int nbk = ns == 1 ? s.Tk / s.blk : static_cast<int>(std::max<long long>(1, (s.q_pos0 + sel[c + 1] - 1) / 4));
    sws = std::max(sws, qsa_workspace_size(QSA_OP_SELECT_TOPK, s.B, rows, nbk, s.k, s.Hq, s.D, 0));
  }
  int rows = 0;
  for (size_t c = 0; c + 1 < att.size(); ++c) rows = std::max(rows, att[c + 1] - att[c]);
  const size_t aws = std::max<size_t>(16, qsa_workspace_size(QSA_OP_SPARSE_ATTN_PREFILL, s.B, rows, 0, s.k, s.Hq,
                                                               s.D, 0));
  L.sel_ws_bytes = std::max<size_t>(sws, 16);
  L.att_ws_bytes = aws;
  L.sel_ws = take(L.sel_ws_bytes);
  // the attention workspace (query tiles) and the interleaved K/V are never used by one call both
  const size_t kvb = attn_kv_supported(s.Hq, s.Hkv, s.D) ? attn_kv_bytes(s.B, s.Tk, s.Hkv, s.D) : 0;
  L.att_ws = take(std::max(L.att_ws_bytes, kvb));
  L.kv = L.att_ws;
  L.total = off;
  return L;
}

bool valid_shape(const Shape& s) {
  if (s.B < 1 || s.Tq < 1 || s.Tk < 1 || s.Hq < 1 || s.Hkv < 1 || s.D < 1 || s.Hi < 1 || s.Di < 1 || s.k < 1)
    return false;
  if (s.blk != 4 || s.q_pos0 < 0 || s.q_pos0 + s.Tq > s.Tk || s.chunks < 0 || s.sel_chunks < 1) return false;
  return true;
}

// Per-device copy streams and a reusable pool of events; one call enqueues at a time per device.
// They live until the process exits (like the library's other per-device caches).
struct DevState {
  std::mutex mu;
  bool ready = false;
  cudaStream_t cin = nullptr, cout = nullptr;
  std::vector<cudaEvent_t> events;
};
DevState g_state[kMaxDev];

cudaError_t ensure_events(DevState& st, size_t n) {
  while (st.events.size() < n) {
    cudaEvent_t e;
    const cudaError_t err = cudaEventCreateWithFlags(&e, cudaEventDisableTiming);
    if (err != cudaSuccess) return err;
    st.events.push_back(e);
  }
  return cudaSuccess;
}

qsa_status_t cuda_st(cudaError_t e) { return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA; }

}  // namespace
}  // namespace qsa

using namespace qsa;

extern "C" {

size_t qsa_prefill_host_device_bytes(int B, int Tq, int Tk, int Hq, int Hkv, int D, int Hi, int Di, int k_blocks,
                                     int blk, int64_t q_pos0, int rope, int chunks, int sel_chunks) {
  const Shape s{B, Tq, Tk, Hq, Hkv, D, Hi, Di, k_blocks, blk, static_cast<long long>(q_pos0), rope != 0, chunks,
                sel_chunks};
  if (!valid_shape(s)) return 0;
  return layout(s).total;
}

qsa_status_t qsa_prefill_host(const void* q_h, const void* k_h, const void* v_h, const void* qi_h, const void* ki_h,
                              void* out_h, int B, int Tq, int Tk, int Hq, int Hkv, int D, int Hi, int Di,
                              int k_blocks, int blk, int64_t q_pos0, float scale, qsa_score_mode_t mode,
                              const float* head_w, const qsa_rope_params_t* rope, int chunks, int sel_chunks,
                              void* dev, size_t dev_bytes, int32_t* idx_out, float* lse_out, void* stream) {
  QSA_NVTX();
  if (!q_h || !k_h || !v_h || !qi_h || !ki_h || !out_h || !dev) return QSA_ERR_INVALID_ARGUMENT;
  if (reinterpret_cast<uintptr_t>(dev) % kAlign != 0 || !(scale > 0.f)) return QSA_ERR_INVALID_ARGUMENT;
  const bool rot = rope != nullptr && rope->theta > 0.0;
  const Shape s{B, Tq, Tk, Hq, Hkv, D, Hi, Di, k_blocks, blk, static_cast<long long>(q_pos0), rot, chunks,
                sel_chunks};
  if (!valid_shape(s)) return QSA_ERR_INVALID_ARGUMENT;
  const Layout L = layout(s);
  if (dev_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDev) return QSA_ERR_CUDA;
  DevState& st = g_state[device];
  std::lock_guard<std::mutex> lk(st.mu);
  if (!st.ready) {
    if (cudaStreamCreateWithFlags(&st.cin, cudaStreamNonBlocking) != cudaSuccess) return QSA_ERR_CUDA;
    if (cudaStreamCreateWithFlags(&st.cout, cudaStreamNonBlocking) != cudaSuccess) return QSA_ERR_CUDA;
    st.ready = true;
  }
  std::vector<int> att, sel;
  chunk_bounds(s, att, sel);
  const int n = static_cast<int>(att.size()) - 1, ns = static_cast<int>(sel.size()) - 1;
  if (cudaError_t e = ensure_events(st, static_cast<size_t>(2 * n + ns + 2)); e != cudaSuccess) return cuda_st(e);
  cudaEvent_t* ev = st.events.data();
  cudaEvent_t ev_start = ev[0], ev_done = ev[1];
  cudaEvent_t* ev_sel = ev + 2;            // [ns] indexer inputs of selection chunk c have arrived
  cudaEvent_t* ev_arr = ev_sel + ns;       // [n] q / K / V of attention chunk c have arrived
  cudaEvent_t* ev_out = ev_arr + n;        // [n] attention of chunk c is done
  cudaStream_t main = static_cast<cudaStream_t>(stream);

  uint8_t* base = static_cast<uint8_t*>(dev);
  uint16_t* q_d = reinterpret_cast<uint16_t*>(base + L.q);
  uint16_t* k_d = reinterpret_cast<uint16_t*>(base + L.k);
  uint16_t* v_d = reinterpret_cast<uint16_t*>(base + L.v);
  uint16_t* qi_d = reinterpret_cast<uint16_t*>(base + L.qi);
  uint16_t* ki_d = reinterpret_cast<uint16_t*>(base + L.ki);
  uint16_t* kp_d = reinterpret_cast<uint16_t*>(base + L.kp);
  uint16_t* qr_d = rot ? reinterpret_cast<uint16_t*>(base + L.qr) : qi_d;
  uint16_t* out_d = reinterpret_cast<uint16_t*>(base + L.out);
  int32_t* idx_d = idx_out ? idx_out : reinterpret_cast<int32_t*>(base + L.idx);
  float* lse_d = lse_out ? lse_out : reinterpret_cast<float*>(base + L.lse);
  void* sel_ws = base + L.sel_ws;
  void* att_ws = base + L.att_ws;
  const bool use_kv = attn_path() == 0 && attn_kv_supported(Hq, Hkv, D) && B <= 65535;
  void* kv_d = base + L.kv;
  long long kv_done_i = 0;   // positions interleaved so far (the block holding it is rewritten next)
  const char* qh = static_cast<const char*>(q_h);
  const char* kh = static_cast<const char*>(k_h);
  const char* vh = static_cast<const char*>(v_h);
  const char* qih = static_cast<const char*>(qi_h);
  const char* kih = static_cast<const char*>(ki_h);
  char* oh = static_cast<char*>(out_h);

  // bytes of one row of each tensor (row = one position of one sequence); with B > 1 there is one
  // chunk and every copy covers whole tensors
  const size_t q_row = static_cast<size_t>(Hq) * D * 2, kv_row = static_cast<size_t>(Hkv) * D * 2;
  const size_t qi_row = static_cast<size_t>(Hi) * Di * 2, ki_row = static_cast<size_t>(Di) * 2;
  auto h2d = [&](void* d, const char* h, size_t off, size_t bytes) {
    return bytes ? cudaMemcpyAsync(static_cast<char*>(d) + off, h + off, bytes, cudaMemcpyHostToDevice, st.cin)
                 : cudaSuccess;
  };
  const size_t Bz = static_cast<size_t>(B);

  // ---------------------------------------------------------------- copies in (stream cin)
  // the device buffers may still be read by earlier work on the caller's stream
  if (cudaError_t e = cudaEventRecord(ev_start, main); e != cudaSuccess) return cuda_st(e);
  if (cudaError_t e = cudaStreamWaitEvent(st.cin, ev_start, 0); e != cudaSuccess) return cuda_st(e);
  for (int c = 0; c < ns; ++c) {
    const long long slo = sel[c], shi = sel[c + 1];
    const long long klo = c ? q_pos0 + slo : 0, khi = c < ns - 1 ? q_pos0 + shi : Tk;
    cudaError_t e = h2d(ki_d, kih, klo * ki_row * Bz, (khi - klo) * ki_row * Bz);
    if (e == cudaSuccess) e = h2d(qi_d, qih, slo * qi_row * Bz, (shi - slo) * qi_row * Bz);
    if (e == cudaSuccess) e = cudaEventRecord(ev_sel[c], st.cin);
    if (e != cudaSuccess) return cuda_st(e);
  }
  long long kv_done = 0;
  for (int c = 0; c < n; ++c) {
    const long long lo = att[c], hi = att[c + 1];
    const long long kv_end = c == n - 1 ? Tk : std::min<long long>(Tk, q_pos0 + hi);
    cudaError_t e = cudaSuccess;
    if (kv_end > kv_done) {
      e = h2d(k_d, kh, kv_done * kv_row * Bz, (kv_end - kv_done) * kv_row * Bz);
      if (e == cudaSuccess) e = h2d(v_d, vh, kv_done * kv_row * Bz, (kv_end - kv_done) * kv_row * Bz);
      kv_done = kv_end;
    }
    if (e == cudaSuccess) e = h2d(q_d, qh, lo * q_row * Bz, (hi - lo) * q_row * Bz);
    if (e == cudaSuccess) e = cudaEventRecord(ev_arr[c], st.cin);
    if (e != cudaSuccess) return cuda_st(e);
  }

  // ---------------------------------------------------------------- pooling + selection (caller's stream)
  for (int c = 0; c < ns; ++c) {
    if (cudaError_t e = cudaStreamWaitEvent(main, ev_sel[c], 0); e != cudaSuccess) return cuda_st(e);
    const int slo = sel[c], shi = sel[c + 1];
    qsa_status_t r;
    if (ns == 1) {
      r = qsa_pool_block_keys_rope(ki_d, kp_d, B, Tk, Di, blk, rot ? rope : nullptr, 0,
                                   static_cast<int64_t>(Tk) * Di, static_cast<int64_t>(Tk / blk) * Di, stream);
      if (r == QSA_OK && rot) r = qsa_rope_index_queries_rope(qi_d, qr_d, B, Tq, Hi, Di, q_pos0, nullptr, rope, stream);
      if (r == QSA_OK)
        r = qsa_select_topk(nullptr, 0, qr_d, kp_d, head_w, nullptr, B, Tq, Tk / blk, Hi, Di, blk, q_pos0, mode,
                            k_blocks, idx_d, sel_ws, L.sel_ws_bytes, stream);
    } else {
      // keys of positions [klo, khi) pool into blocks [klo / 4, khi / 4); the chunk's rows select
      // among the blocks below (q_pos0 + shi - 1) / 4
      const long long klo = c ? q_pos0 + slo : 0, khi = c < ns - 1 ? q_pos0 + shi : Tk;
      r = QSA_OK;
      if (khi / 4 > klo / 4)
        r = qsa_pool_block_keys_rope(ki_d + klo * Di, kp_d + (klo / 4) * Di, 1, static_cast<int>(khi / 4 * 4 - klo),
                                     Di, blk, rot ? rope : nullptr, klo, 0, 0, stream);
      uint16_t* qc = qi_d + static_cast<size_t>(slo) * Hi * Di;
      uint16_t* qrc = qr_d + static_cast<size_t>(slo) * Hi * Di;
      if (r == QSA_OK && rot)
        r = qsa_rope_index_queries_rope(qc, qrc, 1, shi - slo, Hi, Di, q_pos0 + slo, nullptr, rope, stream);
      const int nbk = static_cast<int>(std::max<long long>(1, (q_pos0 + shi - 1) / 4));
      if (r == QSA_OK)
        r = qsa_select_topk(nullptr, 0, qrc, kp_d, head_w, nullptr, 1, shi - slo, nbk, Hi, Di, blk, q_pos0 + slo,
                            mode, k_blocks, idx_d + static_cast<size_t>(slo) * k_blocks, sel_ws, L.sel_ws_bytes,
                            stream);
    }
    if (r != QSA_OK) return r;
  }

  // ---------------------------------------------------------------- attention (caller's stream) + copies out (cout)
  for (int c = 0; c < n; ++c) {
    const int lo = att[c], hi = att[c + 1];
    if (hi <= lo) continue;
    if (cudaError_t e = cudaStreamWaitEvent(main, ev_arr[c], 0); e != cudaSuccess) return cuda_st(e);
    // B > 1: one chunk covering every row of every sequence
    const size_t r0 = static_cast<size_t>(lo);
    qsa_status_t r;
    if (use_kv) {
      const long long kv_end = c == n - 1 ? Tk : std::min<long long>(Tk, q_pos0 + hi);
      r = qsa_interleave_kv(k_d, v_d, kv_d, B, Tk, Hkv, D, blk, kv_done_i, kv_end, stream);
      kv_done_i = kv_end;
      if (r == QSA_OK)
        r = qsa_sparse_attn_prefill_kv(q_d + r0 * Hq * D, kv_d, idx_d + r0 * k_blocks, B, hi - lo, Tk, Hq, Hkv, D,
                                       k_blocks, blk, q_pos0 + lo, scale, out_d + r0 * Hq * D, lse_d + r0 * Hq,
                                       stream);
    } else {
      r = qsa_sparse_attn_prefill_ws(q_d + r0 * Hq * D, k_d, v_d, idx_d + r0 * k_blocks, B, hi - lo, Tk, Hq, Hkv, D,
                                     k_blocks, blk, q_pos0 + lo, scale, out_d + r0 * Hq * D, lse_d + r0 * Hq, att_ws,
                                     L.att_ws_bytes, stream);
    }
    if (r != QSA_OK) return r;
    cudaError_t e = cudaEventRecord(ev_out[c], main);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st.cout, ev_out[c], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(oh + r0 * q_row * Bz, reinterpret_cast<char*>(out_d) + r0 * q_row * Bz,
                          static_cast<size_t>(hi - lo) * q_row * Bz, cudaMemcpyDeviceToHost, st.cout);
    if (e != cudaSuccess) return cuda_st(e);
  }
  // the caller's stream is done with the call once the last output row has arrived in host memory
  cudaError_t e = cudaEventRecord(ev_done, st.cout);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(main, ev_done, 0);
  return cuda_st(e);
}

}  // extern "C"
