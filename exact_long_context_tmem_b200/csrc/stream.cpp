// Chunk streamer: exact attention over host-resident Q/K/V under a device-memory budget.
//
// Stream-CQSA summary, "Methodology" 2-4: attention is split into independent sub-attention
// tasks that together cover every (query, key) pair exactly once; a scheduler queues them,
// streams their inputs into device memory, swaps finished results out to host memory, and a
// light controller sizes the blocks from the memory budget.  Here a task is a (query block,
// key chunk) rectangle of the causal plane; its result is merged into the block's running
// (O, LSE) by the exact log-sum-exp merge inside the prefill kernel's epilogue, and the block is
// copied back when its last task is merged.
//
// Pipeline: K/V chunks and Q blocks are double-buffered; the copy stream loads task t+1 while
// the compute stream runs task t, and finished blocks go back to the host on a third stream, so
// the two directions of the host link overlap each other and the compute; events order buffer
// reuse.  Everything the call allocates on the device counts against the budget and is freed
// before it returns.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdint>
#include <vector>

#include "../../include/attn.h"
#include "internal.h"

namespace {

std::atomic<int> g_inject_what{0};
std::atomic<long long> g_inject_nth{0};

struct Sizes {
  long long q_row, kv_row;  // bytes per token row (all heads, one batch element)
};

Sizes row_sizes(const attn_dims_t& d) {
  return {(long long)d.Hq * d.D * 2, (long long)d.Hkv * d.D * 2};
}

// Device bytes of a plan with query block Bq and key chunk Ck.
long long plan_bytes(const attn_dims_t& d, long long Bq, long long Ck) {
  const long long B = d.B;
  const long long qrows = B * Bq * d.Hq;  // output rows of one block
  const long long q_blk = qrows * d.D * 2;
  const long long kv = B * Ck * d.Hkv * d.D * 2;
  const long long o32 = qrows * d.D * 4;
  const long long l32 = qrows * 4;
  return 2 * q_blk      // Q block, double-buffered
         + 4 * kv       // K and V chunks, double-buffered
         + o32 + l32    // running (O, LSE) of the block, merged into by every task
         + q_blk + l32;  // bf16 O and LSE staged for the copy back
}

// Key chunks a query block [q0, q1) needs: all of them, or (causal) those whose first key is at or
// before the block's last query position.
long long tasks_of_block(long long S, int causal, long long Ck, long long q1) {
  if (!causal) return (S + Ck - 1) / Ck;
  return std::min((S + Ck - 1) / Ck, (q1 - 1) / Ck + 1);
}

struct Guard {
  std::vector<void*> dev;
  std::vector<cudaEvent_t> events;
  cudaStream_t own[3] = {nullptr, nullptr, nullptr};
  ~Guard() {
    for (void* p : dev) cudaFree(p);
    for (cudaEvent_t e : events) cudaEventDestroy(e);
    for (cudaStream_t s : own)
      if (s) cudaStreamDestroy(s);
  }
};

}  // namespace

extern "C" {

attn_status_t attn_debug_inject(int what, long long nth) {
  if (what < 0 || what > 2 || (what != 0 && nth < 1)) return ATTN_ERR_INVALID_ARG;
  g_inject_nth.store(nth);
  g_inject_what.store(what);
  return ATTN_OK;
}

attn_status_t attn_stream_plan(attn_dims_t d, long long S, int causal, long long chunk_tokens,
                               size_t device_budget_bytes, attn_stream_plan_t* plan) {
  if (!plan || d.B <= 0 || d.Hq <= 0 || d.Hkv <= 0 || d.Hq % d.Hkv || S <= 0 || chunk_tokens < 0 ||
      chunk_tokens % 128 || !(d.scale > 0.f))
    return ATTN_ERR_INVALID_ARG;
  if (d.D != 64 && d.D != 128) return ATTN_ERR_UNSUPPORTED;
  const long long budget = (long long)std::min<size_t>(device_budget_bytes, (size_t)1 << 62);
  const long long S128 = (S + 127) / 128 * 128;
  long long Ck = chunk_tokens > 0 ? std::min(chunk_tokens, S128) : std::min<long long>(65536, S128);
  // Shrink the chunk until the smallest plan (one 128-row block) fits.
  while (Ck > 128 && plan_bytes(d, 128, Ck) > budget) Ck = std::max<long long>(128, (Ck / 2 + 127) / 128 * 128);
  if (chunk_tokens > 0 && Ck != std::min(chunk_tokens, S128)) return ATTN_ERR_BUDGET;
  if (plan_bytes(d, 128, Ck) > budget) return ATTN_ERR_BUDGET;
  // Query block (a multiple of the chunk, or of 128 below one chunk) that fits and sends the fewest
  // K/V chunks across the host link (every task loads one), the larger block on a tie.
  long long Bq = 128;
  const long long unit = Ck;
  long long best_tasks = -1;
  for (long long cand = ((S + unit - 1) / unit) * unit; cand >= unit; cand -= unit) {
    const long long bq = std::min(cand, S128);
    if (plan_bytes(d, bq, Ck) > budget) continue;
    long long nt = 0;
    for (long long q0 = 0; q0 < S; q0 += bq) nt += tasks_of_block(S, causal, Ck, std::min(S, q0 + bq));
    if (best_tasks < 0 || nt < best_tasks) {
      best_tasks = nt;
      Bq = bq;
    }
  }
  if (Bq < Ck) {
    for (long long cand = std::min(Ck, S128); cand >= 128; cand -= 128)
      if (plan_bytes(d, cand, Ck) <= budget) {
        Bq = cand;
        break;
      }
  }
  long long n = 0;
  for (long long q0 = 0; q0 < S; q0 += Bq) n += tasks_of_block(S, causal, Ck, std::min(S, q0 + Bq));
  plan->q_block = Bq;
  plan->kv_chunk = Ck;
  plan->n_tasks = n;
  plan->device_bytes = plan_bytes(d, Bq, Ck);
  return ATTN_OK;
}

attn_status_t attn_stream_task(const attn_stream_plan_t* plan, long long S, int causal, long long idx,
                               long long* q_start, long long* kv_start) {
  if (!plan || !q_start || !kv_start || idx < 0 || idx >= plan->n_tasks || plan->q_block <= 0 ||
      plan->kv_chunk <= 0)
    return ATTN_ERR_INVALID_ARG;
  for (long long q0 = 0; q0 < S; q0 += plan->q_block) {
    const long long nt = tasks_of_block(S, causal, plan->kv_chunk, std::min(S, q0 + plan->q_block));
    if (idx < nt) {
      *q_start = q0;
      *kv_start = idx * plan->kv_chunk;
      return ATTN_OK;
    }
    idx -= nt;
  }
  return ATTN_ERR_INVALID_ARG;
}

attn_status_t attn_chunked_stream(const void* q_h, const void* k_h, const void* v_h, void* o_h, float* lse_h,
                                  attn_dims_t d, long long S, int causal, long long chunk_tokens,
                                  size_t device_budget_bytes, void* compute_stream, void* copy_stream,
                                  attn_stream_stats_t* stats) {
  const auto t_start = std::chrono::steady_clock::now();
  if (!q_h || !k_h || !v_h || !o_h) return ATTN_ERR_INVALID_ARG;
  attn_stream_plan_t plan;
  attn_status_t st = attn_stream_plan(d, S, causal, chunk_tokens, device_budget_bytes, &plan);
  if (st != ATTN_OK) return st;
  const int inject_what = g_inject_what.exchange(0);
  const long long inject_nth = g_inject_nth.load();
  long long n_h2d = 0, n_alloc = 0;

  Guard g;
  auto dalloc = [&](void** p, long long bytes) -> attn_status_t {
    ++n_alloc;
    if (inject_what == 2 && n_alloc == inject_nth) return ATTN_ERR_INJECTED;
    if (cudaMalloc(p, (size_t)bytes) != cudaSuccess) return ATTN_ERR_CUDA;
    g.dev.push_back(*p);
    return ATTN_OK;
  };
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(compute_stream);
  cudaStream_t xs = reinterpret_cast<cudaStream_t>(copy_stream);
  if (!cs) {
    if (cudaStreamCreateWithFlags(&g.own[0], cudaStreamNonBlocking) != cudaSuccess) return ATTN_ERR_CUDA;
    cs = g.own[0];
  }
  if (!xs) {
    if (cudaStreamCreateWithFlags(&g.own[1], cudaStreamNonBlocking) != cudaSuccess) return ATTN_ERR_CUDA;
    xs = g.own[1];
  }
  // Device-to-host copies get a stream of their own, so they overlap the next uploads.
  if (cudaStreamCreateWithFlags(&g.own[2], cudaStreamNonBlocking) != cudaSuccess) return ATTN_ERR_CUDA;
  cudaStream_t ds = g.own[2];
  const long long B = d.B, Bq = plan.q_block, Ck = plan.kv_chunk;
  const Sizes rs = row_sizes(d);
  const long long q_blk_bytes = B * Bq * rs.q_row;
  const long long kv_bytes = B * Ck * rs.kv_row;
  const long long qrows = B * Bq * d.Hq;
  void *qbuf[2], *kbuf[2], *vbuf[2], *o_acc, *l_acc, *o_bf, *l_out;
  for (int i = 0; i < 2; ++i) {
    if ((st = dalloc(&qbuf[i], q_blk_bytes)) != ATTN_OK) return st;
    if ((st = dalloc(&kbuf[i], kv_bytes)) != ATTN_OK) return st;
    if ((st = dalloc(&vbuf[i], kv_bytes)) != ATTN_OK) return st;
  }
  if ((st = dalloc(&o_acc, qrows * d.D * 4)) != ATTN_OK) return st;
  if ((st = dalloc(&l_acc, qrows * 4)) != ATTN_OK) return st;
  if ((st = dalloc(&o_bf, q_blk_bytes)) != ATTN_OK) return st;
  if ((st = dalloc(&l_out, qrows * 4)) != ATTN_OK) return st;

  auto mk_event = [&](cudaEvent_t* e, bool timing) -> attn_status_t {
    if (cudaEventCreateWithFlags(e, timing ? cudaEventDefault : cudaEventDisableTiming) != cudaSuccess)
      return ATTN_ERR_CUDA;
    g.events.push_back(*e);
    return ATTN_OK;
  };
  cudaEvent_t q_ready[2], q_free[2], kv_ready[2], kv_free[2], out_ready, out_free, t0, t1, t_begin, t_end;
  for (int i = 0; i < 2; ++i) {
    if ((st = mk_event(&q_ready[i], false)) || (st = mk_event(&q_free[i], false)) ||
        (st = mk_event(&kv_ready[i], false)) || (st = mk_event(&kv_free[i], false)))
      return st;
  }
  if ((st = mk_event(&out_ready, false)) || (st = mk_event(&out_free, false)) || (st = mk_event(&t0, true)) ||
      (st = mk_event(&t1, true)) || (st = mk_event(&t_begin, true)) || (st = mk_event(&t_end, true)))
    return st;
  // Timing: a pair of events around every batch of copies and every compute step, on the stream that
  // runs it; summed after the call's last copy.
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> span_h2d, span_d2h, span_comp;
  auto span_begin = [&](std::vector<std::pair<cudaEvent_t, cudaEvent_t>>& v, cudaStream_t s) -> attn_status_t {
    cudaEvent_t a, b;
    attn_status_t e;
    if ((e = mk_event(&a, true)) != ATTN_OK || (e = mk_event(&b, true)) != ATTN_OK) return e;
    v.emplace_back(a, b);
    return cudaEventRecord(a, s) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  };
  auto span_end = [&](std::vector<std::pair<cudaEvent_t, cudaEvent_t>>& v, cudaStream_t s) -> attn_status_t {
    return cudaEventRecord(v.back().second, s) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  };

  long long h2d = 0, d2h = 0;
  // Host->device copy of `rows` token rows starting at `row0` for every batch element into a packed
  // [B, rows, H, D] device buffer.
  auto h2d_rows = [&](void* dst, const void* src, long long row_bytes, long long row0, long long rows) -> attn_status_t {
    ++n_h2d;
    if (inject_what == 1 && n_h2d == inject_nth) return ATTN_ERR_INJECTED;
    const char* s = static_cast<const char*>(src) + row0 * row_bytes;
    if (cudaMemcpy2DAsync(dst, (size_t)(rows * row_bytes), s, (size_t)(S * row_bytes), (size_t)(rows * row_bytes),
                          (size_t)B, cudaMemcpyHostToDevice, xs) != cudaSuccess)
      return ATTN_ERR_CUDA;
    h2d += B * rows * row_bytes;
    return ATTN_OK;
  };
  auto d2h_rows = [&](void* dst, const void* src, long long row_bytes, long long row0, long long rows) -> attn_status_t {
    char* dd = static_cast<char*>(dst) + row0 * row_bytes;
    if (cudaMemcpy2DAsync(dd, (size_t)(S * row_bytes), src, (size_t)(rows * row_bytes), (size_t)(rows * row_bytes),
                          (size_t)B, cudaMemcpyDeviceToHost, ds) != cudaSuccess)
      return ATTN_ERR_CUDA;
    d2h += B * rows * row_bytes;
    return ATTN_OK;
  };

  auto run = [&]() -> attn_status_t {
    attn_status_t s2;
    if (cudaEventRecord(t_begin, xs) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaStreamWaitEvent(cs, t_begin, 0) != cudaSuccess || cudaStreamWaitEvent(ds, t_begin, 0) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (cudaEventRecord(t0, cs) != cudaSuccess) return ATTN_ERR_CUDA;
    long long task = 0;
    int blk = 0;
    for (long long q0 = 0; q0 < S; q0 += Bq, ++blk) {
      const long long q1 = std::min(S, q0 + Bq), rows = q1 - q0;
      const int qb = blk & 1;
      if (blk == 0) {  // the first Q block; later ones are prefetched during the previous block
        if ((s2 = span_begin(span_h2d, xs)) != ATTN_OK) return s2;
        if ((s2 = h2d_rows(qbuf[0], q_h, rs.q_row, q0, rows)) != ATTN_OK) return s2;
        if ((s2 = span_end(span_h2d, xs)) != ATTN_OK) return s2;
        if (cudaEventRecord(q_ready[0], xs) != cudaSuccess) return ATTN_ERR_CUDA;
      }
      const long long nt = tasks_of_block(S, causal, Ck, q1);
      for (long long j = 0; j < nt; ++j, ++task) {
        const long long k0 = j * Ck, k1 = std::min(S, k0 + Ck), klen = k1 - k0;
        const int kb = (int)(task & 1);
        if (task >= 2 && cudaStreamWaitEvent(xs, kv_free[kb], 0) != cudaSuccess) return ATTN_ERR_CUDA;
        if ((s2 = span_begin(span_h2d, xs)) != ATTN_OK) return s2;
        if ((s2 = h2d_rows(kbuf[kb], k_h, rs.kv_row, k0, klen)) != ATTN_OK) return s2;
        if ((s2 = h2d_rows(vbuf[kb], v_h, rs.kv_row, k0, klen)) != ATTN_OK) return s2;
        if ((s2 = span_end(span_h2d, xs)) != ATTN_OK) return s2;
        if (cudaEventRecord(kv_ready[kb], xs) != cudaSuccess) return ATTN_ERR_CUDA;
        if (j == nt - 1 && q1 < S) {
          // prefetch the next Q block into the other buffer once its previous user is done
          const long long n0 = q1, n1 = std::min(S, q1 + Bq);
          if (blk >= 1 && cudaStreamWaitEvent(xs, q_free[qb ^ 1], 0) != cudaSuccess) return ATTN_ERR_CUDA;
          if ((s2 = span_begin(span_h2d, xs)) != ATTN_OK) return s2;
          if ((s2 = h2d_rows(qbuf[qb ^ 1], q_h, rs.q_row, n0, n1 - n0)) != ATTN_OK) return s2;
          if ((s2 = span_end(span_h2d, xs)) != ATTN_OK) return s2;
          if (cudaEventRecord(q_ready[qb ^ 1], xs) != cudaSuccess) return ATTN_ERR_CUDA;
        }
        if (j == 0 && cudaStreamWaitEvent(cs, q_ready[qb], 0) != cudaSuccess) return ATTN_ERR_CUDA;
        if (cudaStreamWaitEvent(cs, kv_ready[kb], 0) != cudaSuccess) return ATTN_ERR_CUDA;
        if ((s2 = span_begin(span_comp, cs)) != ATTN_OK) return s2;
        attn_dims_t dd = d;
        if (j == 0) {  // the block's first task starts its running (O, LSE)
          s2 = attn_prefill(qbuf[qb], kbuf[kb], vbuf[kb], o_acc, ATTN_F32, static_cast<float*>(l_acc), dd, (int)rows,
                            (int)klen, causal, q0, k0, nullptr, cs);
        } else {       // later tasks merge into it inside the kernel's epilogue
          s2 = attn::prefill_accumulate_f32(qbuf[qb], kbuf[kb], vbuf[kb], static_cast<float*>(o_acc),
                                            static_cast<float*>(l_acc), dd, (int)rows, (int)klen, causal, q0, k0, cs);
        }
        if (s2 != ATTN_OK) return s2;
        if ((s2 = span_end(span_comp, cs)) != ATTN_OK) return s2;
        if (cudaEventRecord(kv_free[kb], cs) != cudaSuccess) return ATTN_ERR_CUDA;
      }
      if (cudaEventRecord(q_free[qb], cs) != cudaSuccess) return ATTN_ERR_CUDA;
      // finished block: (O, LSE) -> bf16 O + LSE staging -> host
      if (blk >= 1 && cudaStreamWaitEvent(cs, out_free, 0) != cudaSuccess) return ATTN_ERR_CUDA;
      if ((s2 = span_begin(span_comp, cs)) != ATTN_OK) return s2;
      s2 = attn_merge_lse(static_cast<float*>(o_acc), static_cast<float*>(l_acc), 1, B * rows * d.Hq, d.D, o_bf,
                          ATTN_BF16, static_cast<float*>(l_out), 0, cs);
      if (s2 != ATTN_OK) return s2;
      if ((s2 = span_end(span_comp, cs)) != ATTN_OK) return s2;
      if (cudaEventRecord(out_ready, cs) != cudaSuccess) return ATTN_ERR_CUDA;
      if (cudaStreamWaitEvent(ds, out_ready, 0) != cudaSuccess) return ATTN_ERR_CUDA;
      if ((s2 = span_begin(span_d2h, ds)) != ATTN_OK) return s2;
      if ((s2 = d2h_rows(o_h, o_bf, rs.q_row, q0, rows)) != ATTN_OK) return s2;
      if (lse_h && (s2 = d2h_rows(lse_h, l_out, (long long)d.Hq * 4, q0, rows)) != ATTN_OK) return s2;
      if ((s2 = span_end(span_d2h, ds)) != ATTN_OK) return s2;
      if (cudaEventRecord(out_free, ds) != cudaSuccess) return ATTN_ERR_CUDA;
    }
    if (cudaEventRecord(t1, cs) != cudaSuccess) return ATTN_ERR_CUDA;
    // the end of the last copy back (the D2H stream runs last)
    if (cudaStreamWaitEvent(ds, t1, 0) != cudaSuccess || cudaEventRecord(t_end, ds) != cudaSuccess)
      return ATTN_ERR_CUDA;
    return ATTN_OK;
  };
  st = run();
  // Whatever happened, let queued work finish before the buffers are freed.
  const cudaError_t e1 = cudaStreamSynchronize(xs);
  const cudaError_t e2 = cudaStreamSynchronize(cs);
  const cudaError_t e3 = cudaStreamSynchronize(ds);
  if (st == ATTN_OK && (e1 != cudaSuccess || e2 != cudaSuccess || e3 != cudaSuccess)) st = ATTN_ERR_CUDA;
  if (st == ATTN_OK) {
    int site = 0;
    const attn_status_t ds = attn_device_status(0, &site);
    if (ds != ATTN_OK) st = ds;
  }
  if (stats) {
    stats->plan = plan;
    stats->h2d_bytes = h2d;
    stats->d2h_bytes = d2h;
    auto elapsed = [&](cudaEvent_t a, cudaEvent_t b) -> double {
      float ms = 0.f;
      return (st == ATTN_OK && cudaEventElapsedTime(&ms, a, b) == cudaSuccess) ? ms : 0.0;
    };
    auto summed = [&](const std::vector<std::pair<cudaEvent_t, cudaEvent_t>>& v) -> double {
      double t = 0.0;
      for (const auto& e : v) t += elapsed(e.first, e.second);
      return t;
    };
    stats->ms_compute = elapsed(t0, t1);
    stats->ms_device = elapsed(t_begin, t_end);
    stats->ms_compute_busy = summed(span_comp);
    stats->ms_h2d = summed(span_h2d);
    stats->ms_d2h = summed(span_d2h);
    stats->ms_total =
        std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t_start).count();
  }
  return st;
}

}  // extern "C"
