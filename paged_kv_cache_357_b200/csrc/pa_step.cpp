// pa_step — one whole paged-cache step from pinned host memory, run by libpa
// itself: upload the step's inputs (one copy), the copy-on-write block
// copies, the cache write of the new tokens, the decode, download the output
// (one copy).  The order is the method's: a shared block is copied before a
// sample writes into it (study notes ch.05 §6.1), a new token is stored
// before the decode reads it (vLLM blog, plain-language section), and the
// decode reaches every block through the tables (vLLM blog §"关键细节" 2).
//
// Per step the host makes one call: no per-field copies, no per-kernel
// launches.  The kernels of a (buffer set, counts) pair are captured once
// into a CUDA graph and replayed; uploads, kernels and downloads sit on three
// streams so that neighbouring steps overlap, ordered by events.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <new>

#include "pa.h"

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxGraphsPerSet = 4;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// fp16 and bf16 alike
constexpr size_t kElemBytes = 2;

bool shape_ok(const pa_step_shape& sh, const pa_pool_desc& pool) {
  if (sh.num_seqs <= 0 || sh.num_q_heads <= 0 || sh.max_blocks_per_seq <= 0 || sh.max_new_tokens < 0 ||
      sh.max_copy_pairs < 0 || pool.num_kv_heads <= 0 || pool.head_dim <= 0 || pool.num_blocks <= 0 ||
      pool.block_size <= 0) {
    return false;
  }
  switch (sh.kind) {
    case PA_STEP_DECODE: return sh.q_len == 1 && sh.max_group_size == 0;
    case PA_STEP_MULTI: return sh.q_len >= 2 && sh.max_group_size == 0;
    case PA_STEP_SHARED_PREFIX: return sh.q_len == 1 && sh.max_group_size >= 1;
    default: return false;
  }
}

// Field sizes in the input block's order; fields a shape does not use are 0.
void layout_of(const pa_step_shape& sh, const pa_pool_desc& pool, pa_step_layout& L) {
  const size_t S = static_cast<size_t>(sh.num_seqs);
  const size_t es = kElemBytes;
  const size_t row = static_cast<size_t>(pool.num_kv_heads) * pool.head_dim * es;
  const size_t T = static_cast<size_t>(sh.max_new_tokens), P = static_cast<size_t>(sh.max_copy_pairs);
  const bool grouped = sh.kind == PA_STEP_SHARED_PREFIX;
  const size_t sizes[9] = {
      S * sh.q_len * sh.num_q_heads * pool.head_dim * es,  // q
      S * sh.max_blocks_per_seq * sizeof(int32_t),         // block_tables
      S * sizeof(int32_t),                                 // seq_lens
      grouped ? (S + 1) * sizeof(int32_t) : 0,             // group_starts
      grouped ? S * sizeof(int32_t) : 0,                   // group_prefix_blocks
      P * 2 * sizeof(int64_t),                             // copy_pairs
      T * row,                                             // new k
      T * row,                                             // new v
      T * sizeof(int64_t),                                 // slot_mapping
  };
  size_t* fields[9] = {&L.q, &L.block_tables, &L.seq_lens, &L.group_starts, &L.group_prefix_blocks,
                       &L.copy_pairs, &L.new_k, &L.new_v, &L.slot_mapping};
  size_t off = 0;
  for (int i = 0; i < 9; ++i) {
    *fields[i] = off;
    off = round_up(off + sizes[i]);
  }
  L.total = off;
  L.out_bytes = sizes[0];
}

}  // namespace

struct pa_step {
  pa_step_shape shape;
  pa_pool_desc pool;
  pa_step_layout layout;
  void* k_pool;
  void* v_pool;
  void* workspace;
  size_t workspace_bytes;
  int32_t* status;
  int num_sets;
  void* din[PA_STEP_MAX_SETS];
  void* hin[PA_STEP_MAX_SETS];
  void* dout[PA_STEP_MAX_SETS];
  void* hout[PA_STEP_MAX_SETS];
  cudaStream_t upload = nullptr, kernels = nullptr, download = nullptr;
  cudaEvent_t uploaded[PA_STEP_MAX_SETS] = {};
  cudaEvent_t computed[PA_STEP_MAX_SETS] = {};
  cudaEvent_t downloaded[PA_STEP_MAX_SETS] = {};
  bool used[PA_STEP_MAX_SETS] = {};
  struct Graph {
    int pairs, tokens, groups;
    cudaGraphExec_t exec;
  };
  Graph graphs[PA_STEP_MAX_SETS][kMaxGraphsPerSet] = {};
  int num_graphs[PA_STEP_MAX_SETS] = {};
  long long steps = 0;
  int pending = -1;  // the set whose download is still to be enqueued

  // Enqueue the download of the pending set.  A step's download is issued
  // with the next step (after that step's upload): a download first waits
  // for its kernels, and an upload queued behind it on the same copy queue
  // would wait too, putting upload, kernels and download of neighbouring
  // steps in series.
  pa_status flush() {
    if (pending < 0) return PA_OK;
    const int k = pending;
    pending = -1;
    if (cudaStreamWaitEvent(download, computed[k], 0) != cudaSuccess ||
        cudaMemcpyAsync(hout[k], dout[k], layout.out_bytes, cudaMemcpyDeviceToHost, download) != cudaSuccess ||
        cudaEventRecord(downloaded[k], download) != cudaSuccess) {
      return PA_ERR_CUDA;
    }
    return PA_OK;
  }

  // The step's kernels on `stream` with set k's buffers (checked by the
  // entry points themselves): the copies and stores of the cache update and
  // the decode, in one launch where the decode's kernel takes them in.
  pa_status launch(int k, int pairs, int tokens, int groups, cudaStream_t stream) const {
    const char* in = static_cast<const char*>(din[k]);
    const pa_step_layout& L = layout;
    pa_cache_update upd{};
    if (pairs > 0) {
      upd.copy_pairs = reinterpret_cast<const int64_t*>(in + L.copy_pairs);
      upd.num_copy_pairs = pairs;
    }
    if (tokens > 0) {
      upd.k = in + L.new_k;
      upd.v = in + L.new_v;
      upd.slot_mapping = reinterpret_cast<const int64_t*>(in + L.slot_mapping);
      upd.num_tokens = tokens;
    }
    const auto* tables = reinterpret_cast<const int32_t*>(in + L.block_tables);
    const auto* lens = reinterpret_cast<const int32_t*>(in + L.seq_lens);
    const pa_step_shape& sh = shape;
    switch (sh.kind) {
      case PA_STEP_MULTI:
        return pa_decode_multi_update(&upd, in + L.q, k_pool, v_pool, tables, sh.max_blocks_per_seq, lens,
                                      sh.num_seqs, sh.q_len, sh.num_q_heads, sh.scale, dout[k], workspace,
                                      workspace_bytes, status, &pool, &sh.opts, stream);
      case PA_STEP_SHARED_PREFIX:
        return pa_decode_shared_prefix_update(&upd, in + L.q, k_pool, v_pool, tables, sh.max_blocks_per_seq, lens,
                                              sh.num_seqs, sh.num_q_heads,
                                              reinterpret_cast<const int32_t*>(in + L.group_starts),
                                              reinterpret_cast<const int32_t*>(in + L.group_prefix_blocks), groups,
                                              sh.max_group_size, sh.scale, dout[k], workspace, workspace_bytes,
                                              status, &pool, &sh.opts, stream);
      default:
        return pa_decode_update(&upd, in + L.q, k_pool, v_pool, tables, sh.max_blocks_per_seq, lens, sh.num_seqs,
                                sh.num_q_heads, sh.scale, dout[k], workspace, workspace_bytes, status, &pool,
                                &sh.opts, stream);
    }
  }

  // Bytes of set k's input block that a step with these counts reads: from
  // the start through the last field it uses.
  size_t upload_bytes(int pairs, int tokens, int groups) const {
    const pa_step_layout& L = layout;
    if (tokens > 0) return L.slot_mapping + static_cast<size_t>(tokens) * sizeof(int64_t);
    if (pairs > 0) return L.copy_pairs + static_cast<size_t>(pairs) * 2 * sizeof(int64_t);
    if (groups > 0) return L.group_prefix_blocks + static_cast<size_t>(groups) * sizeof(int32_t);
    return L.seq_lens + static_cast<size_t>(shape.num_seqs) * sizeof(int32_t);
  }

  // The graph of set k's kernels for these counts, captured on first use.
  pa_status graph_for(int k, int pairs, int tokens, int groups, cudaGraphExec_t* exec) {
    for (int i = 0; i < num_graphs[k]; ++i) {
      const Graph& g = graphs[k][i];
      if (g.pairs == pairs && g.tokens == tokens && g.groups == groups) {
        *exec = g.exec;
        return PA_OK;
      }
    }
    cudaGraph_t graph = nullptr;
    if (cudaStreamBeginCapture(kernels, cudaStreamCaptureModeThreadLocal) != cudaSuccess) return PA_ERR_CUDA;
    const pa_status st = launch(k, pairs, tokens, groups, kernels);
    const cudaError_t end = cudaStreamEndCapture(kernels, &graph);
    if (st != PA_OK || end != cudaSuccess) {
      if (graph != nullptr) cudaGraphDestroy(graph);
      return st != PA_OK ? st : PA_ERR_CUDA;
    }
    cudaGraphExec_t ex = nullptr;
    const cudaError_t inst = cudaGraphInstantiate(&ex, graph, 0);
    cudaGraphDestroy(graph);
    if (inst != cudaSuccess) return PA_ERR_CUDA;
    Graph* slot;
    if (num_graphs[k] < kMaxGraphsPerSet) {
      slot = &graphs[k][num_graphs[k]++];
    } else {  // counts keep changing: replace the oldest
      slot = &graphs[k][0];
      cudaGraphExecDestroy(slot->exec);
      for (int i = 1; i < kMaxGraphsPerSet; ++i) graphs[k][i - 1] = graphs[k][i];
      slot = &graphs[k][kMaxGraphsPerSet - 1];
    }
    *slot = Graph{pairs, tokens, groups, ex};
    *exec = ex;
    return PA_OK;
  }

  void release() {
    if (download != nullptr) flush();
    if (upload != nullptr) cudaStreamSynchronize(upload);
    if (kernels != nullptr) cudaStreamSynchronize(kernels);
    if (download != nullptr) cudaStreamSynchronize(download);
    for (int k = 0; k < PA_STEP_MAX_SETS; ++k) {
      for (int i = 0; i < num_graphs[k]; ++i) cudaGraphExecDestroy(graphs[k][i].exec);
      num_graphs[k] = 0;
      for (cudaEvent_t* e : {&uploaded[k], &computed[k], &downloaded[k]}) {
        if (*e != nullptr) cudaEventDestroy(*e);
        *e = nullptr;
      }
    }
    for (cudaStream_t* s : {&upload, &kernels, &download}) {
      if (*s != nullptr) cudaStreamDestroy(*s);
      *s = nullptr;
    }
  }
};

extern "C" pa_status pa_step_layout_of(const pa_step_shape* shape, const pa_pool_desc* pool, pa_step_layout* layout) {
  if (shape == nullptr || pool == nullptr || layout == nullptr || !shape_ok(*shape, *pool)) return PA_ERR_INVALID_ARG;
  layout_of(*shape, *pool, *layout);
  return PA_OK;
}

extern "C" pa_status pa_step_create(const pa_step_shape* shape, const pa_pool_desc* pool, void* k_pool, void* v_pool,
                                    void* workspace, size_t workspace_bytes, int32_t* dev_status, int32_t num_sets,
                                    void* const* dev_inputs, void* const* host_inputs, void* const* dev_outputs,
                                    void* const* host_outputs, pa_step** out) {
  if (out == nullptr) return PA_ERR_INVALID_ARG;
  *out = nullptr;
  if (shape == nullptr || pool == nullptr || !shape_ok(*shape, *pool) || k_pool == nullptr || v_pool == nullptr ||
      num_sets < 2 || num_sets > PA_STEP_MAX_SETS || dev_inputs == nullptr || host_inputs == nullptr ||
      dev_outputs == nullptr || host_outputs == nullptr) {
    return PA_ERR_INVALID_ARG;
  }
  for (int k = 0; k < num_sets; ++k) {
    for (void* p : {dev_inputs[k], host_inputs[k], dev_outputs[k], host_outputs[k]}) {
      if (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) != 0) return PA_ERR_INVALID_ARG;
    }
  }
  pa_step* st = new (std::nothrow) pa_step();
  if (st == nullptr) return PA_ERR_INVALID_ARG;
  st->shape = *shape;
  st->pool = *pool;
  layout_of(*shape, *pool, st->layout);
  st->k_pool = k_pool;
  st->v_pool = v_pool;
  st->workspace = workspace;
  st->workspace_bytes = workspace_bytes;
  st->status = dev_status;
  st->num_sets = num_sets;
  for (int k = 0; k < num_sets; ++k) {
    st->din[k] = dev_inputs[k];
    st->hin[k] = host_inputs[k];
    st->dout[k] = dev_outputs[k];
    st->hout[k] = host_outputs[k];
  }
  bool ok = cudaStreamCreateWithFlags(&st->upload, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&st->kernels, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&st->download, cudaStreamNonBlocking) == cudaSuccess;
  for (int k = 0; ok && k < num_sets; ++k) {
    ok = cudaEventCreateWithFlags(&st->uploaded[k], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&st->computed[k], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&st->downloaded[k], cudaEventDisableTiming) == cudaSuccess;
  }
  if (!ok) {
    st->release();
    delete st;
    return PA_ERR_CUDA;
  }
  *out = st;
  return PA_OK;
}

extern "C" pa_status pa_step_next_set(pa_step* step, int32_t* set) {
  if (step == nullptr || set == nullptr) return PA_ERR_INVALID_ARG;
  const int k = static_cast<int>(step->steps % step->num_sets);
  if (step->used[k] && cudaEventSynchronize(step->uploaded[k]) != cudaSuccess) return PA_ERR_CUDA;
  *set = k;
  return PA_OK;
}

extern "C" pa_status pa_step_run(pa_step* step, int32_t num_copy_pairs, int32_t num_new_tokens, int32_t num_groups,
                                 int32_t* set) {
  if (step == nullptr) return PA_ERR_INVALID_ARG;
  const pa_step_shape& sh = step->shape;
  if (num_copy_pairs < 0 || num_copy_pairs > sh.max_copy_pairs || num_new_tokens < 0 ||
      num_new_tokens > sh.max_new_tokens || num_groups < 0 ||
      (sh.kind == PA_STEP_SHARED_PREFIX ? (num_groups < 1 || num_groups > sh.num_seqs) : num_groups != 0)) {
    return PA_ERR_INVALID_ARG;
  }
  const int k = static_cast<int>(step->steps % step->num_sets);
  const bool used = step->used[k];
  // upload: after the kernels that last read this set
  if (used && cudaStreamWaitEvent(step->upload, step->computed[k], 0) != cudaSuccess) return PA_ERR_CUDA;
  const size_t bytes = step->upload_bytes(num_copy_pairs, num_new_tokens, num_groups);
  if (cudaMemcpyAsync(step->din[k], step->hin[k], bytes, cudaMemcpyHostToDevice, step->upload) != cudaSuccess ||
      cudaEventRecord(step->uploaded[k], step->upload) != cudaSuccess) {
    return PA_ERR_CUDA;
  }
  // kernels: after this upload and after the download that last read this
  // set's output; the stream keeps them after the previous step's kernels
  if (cudaStreamWaitEvent(step->kernels, step->uploaded[k], 0) != cudaSuccess) return PA_ERR_CUDA;
  if (used && cudaStreamWaitEvent(step->kernels, step->downloaded[k], 0) != cudaSuccess) return PA_ERR_CUDA;
  pa_status st;
  if (step->steps == 0) {
    // the first step runs directly: it sets the kernels' attributes and
    // caches before any capture
    st = step->launch(k, num_copy_pairs, num_new_tokens, num_groups, step->kernels);
  } else {
    cudaGraphExec_t exec = nullptr;
    st = step->graph_for(k, num_copy_pairs, num_new_tokens, num_groups, &exec);
    if (st == PA_OK && cudaGraphLaunch(exec, step->kernels) != cudaSuccess) st = PA_ERR_CUDA;
  }
  if (st != PA_OK) return st;
  if (cudaEventRecord(step->computed[k], step->kernels) != cudaSuccess) return PA_ERR_CUDA;
  // the previous step's download now (behind this step's upload); this
  // step's with the next one, or when its result is waited for
  st = step->flush();
  if (st != PA_OK) return st;
  step->pending = k;
  step->used[k] = true;
  ++step->steps;
  if (set != nullptr) *set = k;
  return PA_OK;
}

extern "C" pa_status pa_step_flush(pa_step* step) {
  if (step == nullptr) return PA_ERR_INVALID_ARG;
  return step->flush();
}

extern "C" pa_status pa_step_wait(pa_step* step, int32_t set) {
  if (step == nullptr || set < 0 || set >= step->num_sets) return PA_ERR_INVALID_ARG;
  if (!step->used[set]) return PA_OK;
  if (step->pending == set) {
    const pa_status st = step->flush();
    if (st != PA_OK) return st;
  }
  return cudaEventSynchronize(step->downloaded[set]) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" pa_status pa_step_synchronize(pa_step* step) {
  if (step == nullptr) return PA_ERR_INVALID_ARG;
  if (step->flush() != PA_OK) return PA_ERR_CUDA;
  const bool ok = cudaStreamSynchronize(step->upload) == cudaSuccess &&
                  cudaStreamSynchronize(step->kernels) == cudaSuccess &&
                  cudaStreamSynchronize(step->download) == cudaSuccess;
  return ok ? PA_OK : PA_ERR_CUDA;
}

extern "C" pa_status pa_step_streams(pa_step* step, void** upload, void** kernels, void** download) {
  if (step == nullptr) return PA_ERR_INVALID_ARG;
  if (upload != nullptr) *upload = step->upload;
  if (kernels != nullptr) *kernels = step->kernels;
  if (download != nullptr) *download = step->download;
  return PA_OK;
}

extern "C" void pa_step_destroy(pa_step* step) {
  if (step == nullptr) return;
  step->release();
  delete step;
}
