// decode.cu - the batch-1 decode step of a Llama-architecture model (model/ and
// inference/ of the ntransformer news summary, "Arquitectura y estructura del
// código"), and the layer-streaming ring (SLEP streaming, "Funciones
// principales": host read, PCIe DMA and GPU compute overlapped with double
// buffering; here pinned host memory -> a two-slot HBM ring on a copy stream).
//
// Per layer, six kernels:
//   1. fused QKV GEMV: RMSNorm(h) prologue, RoPE + fp16 K/V append epilogue
//   2. split-context GQA attention, each split's partial (max, sum, accumulator)
//      to a workspace
//   3. merge of the splits (log-sum-exp rule, fixed order)
//   4. O GEMV, residual add into h
//   5. fused gate/up GEMV: RMSNorm(h) prologue, SwiGLU epilogue
//   6. down GEMV, residual add into h
// plus the step word / RoPE table kernel and the embedding before layer 0 and the
// RMSNorm + LM-head GEMV after the last layer.  Kernels use programmatic dependent
// launch so each one's weight stream starts while the previous one drains; the
// resident step is recorded once as a CUDA graph and replayed, with token and
// position read from device memory.  A verification pass (several tokens, "lanes")
// runs each layer's fused GEMVs once for up to 4 lanes (qmma_multi.cuh: the weights
// streamed once), the attention lane by lane.
#include <chrono>
#include <cstdlib>
#include <cstring>
#include <thread>
#include <vector>

#include "ops.h"
#include "ring.h"

// Formats of one layer's matrices: QKV, O, gate and up, down.
struct ntx_layer_qt {
    int32_t qkv, o, ffn, down;
};

struct ntx_model {
    ntx_model_desc d;
    std::vector<ntx_layer_desc> layers;
    std::vector<ntx_layer_qt> lqt;
    std::vector<uint8_t> skip;   // layers the step leaves out (1), set by ntx_model_set_layer_skip
    int32_t qt_embd = 0, qt_out = 0;
    float* h_prev = nullptr;     // calibration: h before the current layer
    float* cos_dev = nullptr;    // calibration: cosine similarity per layer
    bool calibrating = false;
    int32_t host_path = NTX_HOST_PATH_NONE;   // how streamed layers leave host memory
    // multi-token passes (verification of drafted tokens): per-token hidden states, step
    // words and RoPE tables, drafted and predicted tokens, logits of every token
    float* lane_h = nullptr;
    int32_t* lane_step = nullptr;
    float* lane_rope = nullptr;
    float* lane_act = nullptr;        // [kMaxLanes]: q [n_q head_dim], attention out [same], SwiGLU out [ffn]
    int32_t* spec_tokens = nullptr;   // [2 kMaxLanes]: drafted tokens, then the full model's predictions
    float* spec_logits = nullptr;     // [kMaxLanes, vocab]
    std::vector<void*> registered;            // host ranges this library registered (unregistered at destroy)
    int device = 0;
    float* h = nullptr;
    float* q = nullptr;
    float* att = nullptr;
    float* act = nullptr;
    int32_t* step = nullptr;
    float* rope = nullptr;   // the step's RoPE table [head_dim / 2][cos, sin]
    void* attn_ws = nullptr;
    int n_split = 1;
    bool pdl = true;
    bool use_graph = true;
    // CUDA graph of the resident step
    cudaGraphExec_t graph = nullptr;
    float* graph_logits = nullptr;
    // CUDA graphs of resident verification passes, by token count (1 .. 8), and their logits
    cudaGraphExec_t vgraph[9] = {};
    float* vgraph_logits[9] = {};
    // CUDA graph of a draft step of self-speculative decoding, and the layers it leaves out
    cudaGraphExec_t dgraph = nullptr;
    std::vector<uint8_t> dgraph_also;
    // streaming ring
    uint8_t* ring = nullptr;
    size_t slot_bytes = 0;
    size_t off_qkv = 0, off_o = 0, off_gate = 0, off_up = 0, off_down = 0;
    size_t sz_qkv = 0, sz_o = 0, sz_ffn = 0, sz_down = 0;
    cudaEvent_t copy_done[2] = {nullptr, nullptr};
    cudaEvent_t slot_free[2] = {nullptr, nullptr};
    cudaEvent_t ev_start = nullptr, ev_end = nullptr;
    int64_t last_h2d = 0;
};

namespace ntx {
namespace {

using gemv::Params;

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct LayerW {
    const void *qkv, *o, *gate, *up, *down;
};

// What follows a layer in the step: the next resident layer (-1: none).
struct NextLayer {
    int layer;
};

// The per-token state of a step: hidden state h, the step word (token, pos), the RoPE
// table of pos, and the token's activations (q, attention output, SwiGLU output).  A plain
// step has one; a verification pass has one per token.
struct Lane {
    float* h;
    int32_t* step;
    float* rope;
    float* q;
    float* att;
    float* act;
};

Lane lane0(ntx_model* m) { return {m->h, m->step, m->rope, m->q, m->att, m->act}; }

// The fused GEMV launches of a layer, one function per kind, exactly as the step issues
// them: the parameters of a kind for one lane, then its launch.
Params qkv_params(ntx_model* m, int l, const void* w, bool pdl, const Lane& ln)
{
    const ntx_model_desc& d = m->d;
    const ntx_layer_desc& L = m->layers[l];
    const int qd = d.n_q_heads * d.head_dim, kvd = d.n_kv_heads * d.head_dim;
    Params P{};
    P.W = (const uint8_t*)w;
    P.row_bytes = row_bytes(m->lqt[l].qkv, d.hidden);
    P.M = qd + 2 * kvd;
    P.K = d.hidden;
    P.x = ln.h;
    P.norm_w = L.attn_norm;
    P.eps = d.rms_eps;
    P.q_rows = qd;
    P.kv_rows = kvd;
    P.head_dim = d.head_dim;
    P.max_ctx = d.max_ctx;
    P.pos_dev = ln.step + 1;
    P.rope_cs = ln.rope;
    P.k_cache = (__half*)L.k_cache;
    P.v_cache = (__half*)L.v_cache;
    P.q_out = ln.q;
    P.use_pdl = pdl;
    return P;
}

Params o_params(ntx_model* m, int l, const void* w, bool pdl, const Lane& ln)
{
    const ntx_model_desc& d = m->d;
    Params P{};
    P.W = (const uint8_t*)w;
    P.K = d.n_q_heads * d.head_dim;
    P.row_bytes = row_bytes(m->lqt[l].o, P.K);
    P.M = d.hidden;
    P.x = ln.att;
    P.y = ln.h;
    P.use_pdl = pdl;
    return P;
}

Params gate_up_params(ntx_model* m, int l, const void* wg, const void* wu, bool pdl, const Lane& ln)
{
    const ntx_model_desc& d = m->d;
    Params P{};
    P.W = (const uint8_t*)wg;
    P.W2 = (const uint8_t*)wu;
    P.row_bytes = row_bytes(m->lqt[l].ffn, d.hidden);
    P.M = d.ffn;
    P.K = d.hidden;
    P.x = ln.h;
    P.norm_w = m->layers[l].ffn_norm;
    P.eps = d.rms_eps;
    P.y = ln.act;
    P.use_pdl = pdl;
    return P;
}

Params down_params(ntx_model* m, int l, const void* w, bool pdl, const Lane& ln)
{
    const ntx_model_desc& d = m->d;
    Params P{};
    P.W = (const uint8_t*)w;
    P.row_bytes = row_bytes(m->lqt[l].down, d.ffn);
    P.M = d.hidden;
    P.K = d.ffn;
    P.x = ln.act;
    P.y = ln.h;
    P.use_pdl = pdl;
    return P;
}

Params head_params(ntx_model* m, float* logits, bool pdl, const Lane& ln)
{
    const ntx_model_desc& d = m->d;
    Params P{};
    P.W = (const uint8_t*)d.output;
    P.row_bytes = row_bytes(m->qt_out, d.hidden);
    P.M = d.vocab;
    P.K = d.hidden;
    P.x = ln.h;
    P.norm_w = d.out_norm;
    P.eps = d.rms_eps;
    P.y = logits;
    P.use_pdl = pdl;
    return P;
}

ntx_status launch_qkv(ntx_model* m, int l, const void* w, cudaStream_t s, bool pdl, const Lane& ln)
{
    return gemv_launch(m->lqt[l].qkv, gemv::EPI_QKV, gemv::PRO_RMSNORM, qkv_params(m, l, w, pdl, ln), s);
}

ntx_status launch_o(ntx_model* m, int l, const void* w, cudaStream_t s, bool pdl, const Lane& ln)
{
    return gemv_launch(m->lqt[l].o, gemv::EPI_ADD, gemv::PRO_X, o_params(m, l, w, pdl, ln), s);
}

ntx_status launch_gate_up(ntx_model* m, int l, const void* wg, const void* wu, cudaStream_t s, bool pdl,
                          const Lane& ln)
{
    return gemv_launch(m->lqt[l].ffn, gemv::EPI_SWIGLU, gemv::PRO_RMSNORM, gate_up_params(m, l, wg, wu, pdl, ln),
                       s);
}

ntx_status launch_down(ntx_model* m, int l, const void* w, cudaStream_t s, bool pdl, const Lane& ln)
{
    return gemv_launch(m->lqt[l].down, gemv::EPI_ADD, gemv::PRO_X, down_params(m, l, w, pdl, ln), s);
}

ntx_status launch_attention(ntx_model* m, int l, cudaStream_t s, bool pdl, const Lane& ln,
                            const KvPrefetch* pf = nullptr)
{
    const ntx_model_desc& d = m->d;
    const ntx_layer_desc& L = m->layers[l];
    AttnArgs a{};
    a.q = ln.q;
    a.k_cache = (const __half*)L.k_cache;
    a.v_cache = (const __half*)L.v_cache;
    a.out = ln.att;
    a.n_q_heads = d.n_q_heads;
    a.n_kv_heads = d.n_kv_heads;
    a.head_dim = d.head_dim;
    a.max_ctx = d.max_ctx;
    a.pos_dev = ln.step + 1;
    a.workspace = m->attn_ws;
    a.n_split = m->n_split;
    a.pdl = pdl;
    if (pf) a.pf = *pf;
    return attn_launch(a, s);
}

// Whether a layer's attention launch fetches the next layer's K / V rows into L2
// (NTX_L2_PF=0 turns it off; a tuning override).  Measured on B200: Llama-8B Q8_0 decode
// 493.0 -> 497.2 tok/s, Llama-70B Q6_K level.
bool kv_prefetch_on()
{
    const char* env = std::getenv("NTX_L2_PF");
    return !(env && env[0] == '0');
}

ntx_status enqueue_layer(ntx_model* m, int l, const LayerW& w, cudaStream_t s, bool pdl, const Lane& ln,
                         const NextLayer* next = nullptr)
{
    const ntx_model_desc& d = m->d;
    ntx_status st;
    if (m->calibrating) {
        // h before the layer, for the similarity of its input and output
        NTX_CUDA_TRY(cudaMemcpyAsync(m->h_prev, ln.h, (size_t)d.hidden * 4, cudaMemcpyDeviceToDevice, s));
        pdl = false;
    }
    KvPrefetch pf{};
    if (kv_prefetch_on() && next && next->layer >= 0) {
        pf.k = (const uint8_t*)m->layers[next->layer].k_cache;
        pf.v = (const uint8_t*)m->layers[next->layer].v_cache;
        pf.n_kv = d.n_kv_heads;
        pf.row_b = d.head_dim * 2;
        pf.head_stride = (int64_t)d.max_ctx * d.head_dim * 2;
    }
    if ((st = launch_qkv(m, l, w.qkv, s, pdl, ln)) != NTX_OK) return st;
    if ((st = launch_attention(m, l, s, pdl, ln, &pf)) != NTX_OK) return st;
    if ((st = launch_o(m, l, w.o, s, pdl, ln)) != NTX_OK) return st;
    if ((st = launch_gate_up(m, l, w.gate, w.up, s, pdl, ln)) != NTX_OK) return st;
    if ((st = launch_down(m, l, w.down, s, pdl, ln)) != NTX_OK) return st;
    if (m->calibrating) return cosine_launch(m->h_prev, ln.h, d.hidden, m->cos_dev + l, s);
    return NTX_OK;
}

ntx_status enqueue_head(ntx_model* m, float* logits, cudaStream_t s, bool pdl, const Lane& ln)
{
    return gemv_launch(m->qt_out, gemv::EPI_STORE, gemv::PRO_RMSNORM, head_params(m, logits, pdl, ln), s);
}

// One fused GEMV kind over n lanes (params(i): the kind's parameters for lane i): launches
// of up to 4 lanes each that stream the weights once (tiled formats, when the lanes' x fit
// in shared memory), else one launch per lane.  NTX_VERIFY_PER_TOKEN=1 in the environment
// keeps one launch per lane (a test and tuning override).
template <typename ParamsOf>
ntx_status launch_lanes(int qt, int epi, int pro, int n, ParamsOf params, cudaStream_t s)
{
    const char* env = std::getenv("NTX_VERIFY_PER_TOKEN");
    const bool per_token = env && env[0] && env[0] != '0';
    int i = 0;
    while (i < n) {
        int done = 0;
        for (int c = std::min(gemv::kMaxVecs, n - i); c >= 2 && !per_token && !done; --c) {
            const Params P = params(i);
            gemv::Vecs V{};
            for (int v = 0; v < c; ++v) {
                const Params Pv = params(i + v);
                V.x[v] = Pv.x;
                V.y[v] = Pv.y;
                V.q_out[v] = Pv.q_out;
                V.pos_dev[v] = Pv.pos_dev;
                V.rope_cs[v] = Pv.rope_cs;
            }
            const ntx_status st = gemv_multi_launch(qt, epi, pro, P, V, c, s);
            if (st == NTX_OK) done = c;
            else if (st != NTX_EUNSUPPORTED) return st;
        }
        if (!done) {
            const ntx_status st = gemv_launch(qt, epi, pro, params(i), s);
            if (st != NTX_OK) return st;
            done = 1;
        }
        i += done;
    }
    return NTX_OK;
}

// Layer l for n lanes (a verification pass): each fused GEMV kind once for all lanes (the
// weights streamed once per launch of up to 4 lanes), the attention lane by lane.  All
// lanes' K / V rows are written before any lane's attention runs, and lane i reads rows
// 0 .. pos_i only, so lane i sees the rows of lanes 0 .. i as in one-token steps.
// The GEMVs may launch as programmatic dependents (pdl): what they read before their wait
// (weights, norm weights, the lanes' RoPE tables) was written before the pass.  The
// attention never does here: its producer prefetches every row but the newest before its
// wait, and in a pass the rows of the earlier lanes are written by this layer's QKV launch.
ntx_status enqueue_layer_lanes(ntx_model* m, int l, const LayerW& w, cudaStream_t s, bool pdl, const Lane* lanes,
                               int n, const NextLayer* next = nullptr)
{
    if (n == 1) return enqueue_layer(m, l, w, s, pdl, lanes[0], next);
    const ntx_layer_qt& q = m->lqt[l];
    ntx_status st;
    if ((st = launch_lanes(q.qkv, gemv::EPI_QKV, gemv::PRO_RMSNORM, n,
                           [&](int i) { return qkv_params(m, l, w.qkv, pdl, lanes[i]); }, s)) != NTX_OK)
        return st;
    for (int i = 0; i < n; ++i)
        if ((st = launch_attention(m, l, s, false, lanes[i])) != NTX_OK) return st;
    if ((st = launch_lanes(q.o, gemv::EPI_ADD, gemv::PRO_X, n,
                           [&](int i) { return o_params(m, l, w.o, pdl, lanes[i]); }, s)) != NTX_OK)
        return st;
    if ((st = launch_lanes(q.ffn, gemv::EPI_SWIGLU, gemv::PRO_RMSNORM, n,
                           [&](int i) { return gate_up_params(m, l, w.gate, w.up, pdl, lanes[i]); }, s)) != NTX_OK)
        return st;
    return launch_lanes(q.down, gemv::EPI_ADD, gemv::PRO_X, n,
                        [&](int i) { return down_params(m, l, w.down, pdl, lanes[i]); }, s);
}

// The heads of n lanes, lane i's logits at logits + i vocab.
ntx_status enqueue_heads(ntx_model* m, float* logits, cudaStream_t s, bool pdl, const Lane* lanes, int n)
{
    if (n == 1) return enqueue_head(m, logits, s, pdl, lanes[0]);
    return launch_lanes(m->qt_out, gemv::EPI_STORE, gemv::PRO_RMSNORM, n,
                        [&](int i) { return head_params(m, logits + (size_t)i * m->d.vocab, pdl, lanes[i]); }, s);
}

LayerW resident_w(const ntx_layer_desc& L) { return {L.w_qkv, L.w_o, L.w_gate, L.w_up, L.w_down}; }

// Whether layer l runs: not in the skip mask (the calibration runs every layer), and not
// in the extra mask `also_skip` (the draft model of a speculative step; may be null).
bool layer_runs(const ntx_model* m, int l, const uint8_t* also_skip)
{
    if (m->calibrating) return true;
    return !m->skip[l] && !(also_skip && also_skip[l]);
}

// Embedding + resident layers [0, n) for every lane (token / pos from each lane's step
// word), then, if logits is not null, the head of each lane into logits + i vocab.  The
// lanes go through a layer one after another, so lane i's attention sees the K / V rows
// lanes 0..i-1 wrote at their positions.
ntx_status enqueue_resident(ntx_model* m, int n, float* logits, cudaStream_t s, const Lane* lanes, int n_lanes,
                            const uint8_t* also_skip = nullptr)
{
    const bool pdl = m->pdl;
    ntx_status st;
    for (int i = 0; i < n_lanes; ++i)
        if ((st = embed_launch(m->qt_embd, m->d.tok_embd, m->d.hidden, lanes[i].step, lanes[i].h, s,
                               pdl && n_lanes == 1)) != NTX_OK)
            return st;
    for (int l = 0; l < n; ++l) {
        if (!layer_runs(m, l, also_skip)) continue;
        // the next resident layer of this call, if any
        int nl = l + 1;
        while (nl < n && !layer_runs(m, nl, also_skip)) ++nl;
        const NextLayer next{nl < n ? nl : -1};
        if ((st = enqueue_layer_lanes(m, l, resident_w(m->layers[l]), s, pdl, lanes, n_lanes, &next)) != NTX_OK)
            return st;
    }
    if (logits) return enqueue_heads(m, logits, s, pdl, lanes, n_lanes);
    return NTX_OK;
}

ntx_status enqueue_resident(ntx_model* m, int n, float* logits, cudaStream_t s, bool with_head)
{
    const Lane ln = lane0(m);
    return enqueue_resident(m, n, with_head ? logits : nullptr, s, &ln, 1);
}

bool env_flag(const char* name)
{
    const char* v = std::getenv(name);
    return v && v[0] && v[0] != '0';
}

// Format of tensor i of the descriptor: 0 tok_embd, 1 output, then 4 per layer.
int32_t tensor_qtype(const ntx_model_desc* d, int i) { return d->tensor_qtypes ? d->tensor_qtypes[i] : d->qtype; }

// A packed matrix of `cols` columns in format qt that a decode-step GEMV can stream.
ntx_status check_matrix_format(int32_t qt, int64_t cols, const char* what)
{
    const std::string w(what);
    if (qtraits(qt).block_elems == 0) return fail(NTX_EINVAL, "model: unknown format for " + w);
    if (qt == NTX_Q5_K) return fail(NTX_EUNSUPPORTED, "model: " + w + ": Q5_K matrices need the tiled layout NTX_Q5_K_T");
    if (row_bytes(qt, cols) == 0) return fail(NTX_EINVAL, "model: " + w + ": row length not a multiple of the block size");
    if (row_bytes(qt, cols) % 16) return fail(NTX_EUNSUPPORTED, "model: " + w + ": packed rows must be multiples of 16 bytes");
    return NTX_OK;
}

// How the streamed layers' matrices leave host memory ("Funciones principales" of the
// ntransformer news summary picks the data path by what the system offers): page-locked
// memory is copied by DMA directly (NTX_HOST_PATH_PINNED); other host memory is
// page-locked in place with cudaHostRegister (NTX_HOST_PATH_REGISTERED; undone at
// destroy); if that is refused, or NTX_NO_HOST_REGISTER is set, the copies go from
// pageable memory (NTX_HOST_PATH_PAGEABLE: the driver stages them, the host waits for
// each).  The model's path is the slowest one any streamed matrix takes.
ntx_status choose_host_path(ntx_model* m)
{
    const ntx_model_desc& d = m->d;
    const char* no_reg = std::getenv("NTX_NO_HOST_REGISTER");
    const bool may_register = !(no_reg && no_reg[0] && no_reg[0] != '0');
    int path = NTX_HOST_PATH_PINNED;
    for (int l = d.n_resident; l < d.n_layers; ++l) {
        size_t b[5];
        const ntx_layer_qt& q = m->lqt[l];
        const int qd = d.n_q_heads * d.head_dim, kvd = d.n_kv_heads * d.head_dim;
        b[0] = (size_t)(qd + 2 * kvd) * row_bytes(q.qkv, d.hidden);
        b[1] = (size_t)d.hidden * row_bytes(q.o, qd);
        b[2] = b[3] = (size_t)d.ffn * row_bytes(q.ffn, d.hidden);
        b[4] = (size_t)d.hidden * row_bytes(q.down, d.ffn);
        const ntx_layer_desc& L = m->layers[l];
        const void* ptrs[5] = {L.w_qkv, L.w_o, L.w_gate, L.w_up, L.w_down};
        for (int k = 0; k < 5; ++k) {
            cudaPointerAttributes a{};
            const cudaError_t e = cudaPointerGetAttributes(&a, ptrs[k]);
            if (e != cudaSuccess) cudaGetLastError();
            const cudaMemoryType t = e == cudaSuccess ? a.type : cudaMemoryTypeUnregistered;
            if (t == cudaMemoryTypeDevice || t == cudaMemoryTypeManaged)
                return fail(NTX_EINVAL, "ntx_model_create: streamed layer " + std::to_string(l) +
                                            " has a matrix in device memory (streamed matrices live in host memory)");
            if (t == cudaMemoryTypeHost) continue;
            bool ok = false;
            if (may_register) {
                ok = cudaHostRegister(const_cast<void*>(ptrs[k]), b[k], cudaHostRegisterReadOnly) == cudaSuccess;
                if (!ok) {
                    cudaGetLastError();
                    ok = cudaHostRegister(const_cast<void*>(ptrs[k]), b[k], cudaHostRegisterDefault) == cudaSuccess;
                    if (!ok) cudaGetLastError();
                }
            }
            if (ok) {
                m->registered.push_back(const_cast<void*>(ptrs[k]));
                path = std::max(path, (int)NTX_HOST_PATH_REGISTERED);
            } else {
                path = NTX_HOST_PATH_PAGEABLE;
            }
        }
    }
    m->host_path = path;
    return NTX_OK;
}

// Shapes and formats of the descriptor (no pointer is looked at).
ntx_status check_shapes(const ntx_model_desc* d)
{
    if (!d) return fail(NTX_EINVAL, "model: null descriptor");
    if (qtraits(d->qtype).block_elems == 0) return fail(NTX_EINVAL, "model: unknown qtype");
    if (d->n_layers < 1 || d->hidden < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1 || d->ffn < 1 || d->vocab < 1)
        return fail(NTX_EINVAL, "model: dimensions must be positive");
    if (d->head_dim != 128) return fail(NTX_EUNSUPPORTED, "model: head_dim must be 128");
    if (d->n_q_heads % d->n_kv_heads) return fail(NTX_EINVAL, "model: n_q_heads must be a multiple of n_kv_heads");
    const int G = d->n_q_heads / d->n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return fail(NTX_EUNSUPPORTED, "model: q heads per kv head must be 1, 2, 4 or 8");
    if (d->n_kv_heads > 64) return fail(NTX_EUNSUPPORTED, "model: at most 64 kv heads");
    if (d->max_ctx < 1) return fail(NTX_EINVAL, "model: max_ctx must be >= 1");
    if (!(d->rms_eps >= 0.f) || !(d->rope_theta > 0.f)) return fail(NTX_EINVAL, "model: bad eps / theta");
    if (d->n_resident < 0 || d->n_resident > d->n_layers) return fail(NTX_EINVAL, "model: n_resident out of range");
    const int qd = d->n_q_heads * d->head_dim;
    for (int64_t k : {(int64_t)d->hidden, (int64_t)qd, (int64_t)d->ffn})
        if (k > 32768) return fail(NTX_EUNSUPPORTED, "model: row length above 32768");
    ntx_status st;
    // the embedding is read one row at a time (any layout); every other matrix is streamed
    if (qtraits(tensor_qtype(d, 0)).block_elems == 0 || row_bytes(tensor_qtype(d, 0), d->hidden) == 0)
        return fail(NTX_EINVAL, "model: bad format for tok_embd");
    if ((st = check_matrix_format(tensor_qtype(d, 1), d->hidden, "output")) != NTX_OK) return st;
    for (int l = 0; l < d->n_layers; ++l) {
        const int b = 2 + 4 * l;
        if ((st = check_matrix_format(tensor_qtype(d, b), d->hidden, "w_qkv")) != NTX_OK ||
            (st = check_matrix_format(tensor_qtype(d, b + 1), qd, "w_o")) != NTX_OK ||
            (st = check_matrix_format(tensor_qtype(d, b + 2), d->hidden, "w_gate / w_up")) != NTX_OK ||
            (st = check_matrix_format(tensor_qtype(d, b + 3), d->ffn, "w_down")) != NTX_OK)
            return st;
    }
    return NTX_OK;
}

ntx_status check_desc(const ntx_model_desc* d)
{
    ntx_status st = check_shapes(d);
    if (st != NTX_OK) return st;
    if (!d->tok_embd || !d->out_norm || !d->output || !d->layers) return fail(NTX_EINVAL, "model: null pointer");
    if (!aligned(d->tok_embd, 16) || !aligned(d->output, 16) || !aligned(d->out_norm, 16))
        return fail(NTX_EINVAL, "model: tensors must be 16-byte aligned");
    for (int l = 0; l < d->n_layers; ++l) {
        const ntx_layer_desc& L = d->layers[l];
        if (!L.attn_norm || !L.ffn_norm || !L.w_qkv || !L.w_o || !L.w_gate || !L.w_up || !L.w_down || !L.k_cache || !L.v_cache)
            return fail(NTX_EINVAL, "model: null layer pointer (layer " + std::to_string(l) + ")");
        if (!aligned(L.w_qkv, 16) || !aligned(L.w_o, 16) || !aligned(L.w_gate, 16) || !aligned(L.w_up, 16) ||
            !aligned(L.attn_norm, 16) || !aligned(L.ffn_norm, 16) ||
            !aligned(L.w_down, 16) || !aligned(L.k_cache, 16) || !aligned(L.v_cache, 16))
            return fail(NTX_EINVAL, "model: tensors must be 16-byte aligned (layer " + std::to_string(l) + ")");
    }
    return NTX_OK;
}

// Bytes of the five packed matrices of layer l, matrix by matrix (QKV, O, gate, up, down).
void layer_matrix_bytes(const ntx_model_desc* d, int l, size_t (&b)[5])
{
    const int qd = d->n_q_heads * d->head_dim, kvd = d->n_kv_heads * d->head_dim, t = 2 + 4 * l;
    b[0] = (size_t)(qd + 2 * kvd) * row_bytes(tensor_qtype(d, t), d->hidden);
    b[1] = (size_t)d->hidden * row_bytes(tensor_qtype(d, t + 1), qd);
    b[2] = b[3] = (size_t)d->ffn * row_bytes(tensor_qtype(d, t + 2), d->hidden);
    b[4] = (size_t)d->hidden * row_bytes(tensor_qtype(d, t + 3), d->ffn);
}

// Bytes of the HBM ring for layers [n_resident, n_layers): two slots, each holding the
// largest of every matrix over those layers (256-byte aligned).
size_t ring_bytes(const ntx_model_desc* d, int n_resident)
{
    if (n_resident >= d->n_layers) return 0;
    size_t mx[5] = {0, 0, 0, 0, 0};
    for (int l = n_resident; l < d->n_layers; ++l) {
        size_t b[5];
        layer_matrix_bytes(d, l, b);
        for (int k = 0; k < 5; ++k) mx[k] = std::max(mx[k], b[k]);
    }
    size_t slot = 0;
    for (int k = 0; k < 5; ++k) slot += align256(mx[k]);
    return 2 * slot;
}

// Device memory the model itself allocates, besides the ring.
size_t scratch_bytes(const ntx_model_desc* d)
{
    const int qd = d->n_q_heads * d->head_dim;
    const size_t ws = attn_workspace_bytes_for(d->n_q_heads, d->n_kv_heads, d->head_dim,
                                               attn_split_for(d->n_q_heads, d->n_kv_heads, d->max_ctx));
    return (size_t)4 * (2 * d->hidden + 2 * qd + d->ffn + d->head_dim + d->n_layers) + 16 + ws;
}

// Everything in HBM with the first n layers resident: embedding and LM-head matrices, norm
// weights, every layer's KV cache, the resident layers' matrices, the ring, the scratch.
size_t hbm_bytes_for(const ntx_model_desc* d, int n)
{
    size_t total = (size_t)d->vocab * row_bytes(tensor_qtype(d, 0), d->hidden) +
                   (size_t)d->vocab * row_bytes(tensor_qtype(d, 1), d->hidden);
    total += (size_t)(2 * d->n_layers + 1) * d->hidden * 4;
    total += (size_t)d->n_layers * 2 * d->n_kv_heads * d->max_ctx * d->head_dim * 2;
    for (int l = 0; l < n; ++l) {
        size_t b[5];
        layer_matrix_bytes(d, l, b);
        total += b[0] + b[1] + b[2] + b[3] + b[4];
    }
    return total + ring_bytes(d, n) + scratch_bytes(d);
}

constexpr int kMaxLanes = 8;   // tokens of one verification pass
static_assert(sizeof(ntx_model::vgraph) / sizeof(cudaGraphExec_t) == kMaxLanes + 1, "one graph per token count");

void free_model(ntx_model* m)
{
    if (!m) return;
    cudaFree(m->lane_h);
    cudaFree(m->lane_step);
    cudaFree(m->lane_rope);
    cudaFree(m->lane_act);
    cudaFree(m->spec_tokens);
    cudaFree(m->spec_logits);
    for (void* p : m->registered) cudaHostUnregister(p);
    if (m->graph) cudaGraphExecDestroy(m->graph);
    for (cudaGraphExec_t g : m->vgraph)
        if (g) cudaGraphExecDestroy(g);
    if (m->dgraph) cudaGraphExecDestroy(m->dgraph);
    for (int i = 0; i < 2; ++i) {
        if (m->copy_done[i]) cudaEventDestroy(m->copy_done[i]);
        if (m->slot_free[i]) cudaEventDestroy(m->slot_free[i]);
    }
    if (m->ev_start) cudaEventDestroy(m->ev_start);
    if (m->ev_end) cudaEventDestroy(m->ev_end);
    cudaFree(m->h);
    cudaFree(m->q);
    cudaFree(m->att);
    cudaFree(m->act);
    cudaFree(m->step);
    cudaFree(m->rope);
    cudaFree(m->h_prev);
    cudaFree(m->cos_dev);
    cudaFree(m->attn_ws);
    cudaFree(m->ring);
    delete m;
}

}  // namespace

cudaError_t take_device_error_decode(uint32_t* out) { return take_tu_device_error(out); }

}  // namespace ntx

using namespace ntx;

NTX_EXPORT ntx_status ntx_model_create(const ntx_model_desc* desc, ntx_model** model)
{
    if (!model) return fail(NTX_EINVAL, "ntx_model_create: null output pointer");
    *model = nullptr;
    ntx_status st = check_desc(desc);
    if (st != NTX_OK) return st;
    ntx_model* m = new ntx_model();
    m->d = *desc;
    m->layers.assign(desc->layers, desc->layers + desc->n_layers);
    m->d.layers = nullptr;
    m->d.tensor_qtypes = nullptr;
    m->skip.assign(desc->n_layers, 0);
    m->qt_embd = tensor_qtype(desc, 0);
    m->qt_out = tensor_qtype(desc, 1);
    for (int l = 0; l < desc->n_layers; ++l) {
        const int b = 2 + 4 * l;
        m->lqt.push_back({tensor_qtype(desc, b), tensor_qtype(desc, b + 1), tensor_qtype(desc, b + 2),
                          tensor_qtype(desc, b + 3)});
    }
    cudaGetDevice(&m->device);
    const ntx_model_desc& d = m->d;
    const int qd = d.n_q_heads * d.head_dim;
    m->pdl = !env_flag("NTX_NO_PDL");
    m->use_graph = !env_flag("NTX_NO_GRAPH");
    m->n_split = attn_split_for(d.n_q_heads, d.n_kv_heads, d.max_ctx);
    const size_t ws = attn_workspace_bytes_for(d.n_q_heads, d.n_kv_heads, d.head_dim, m->n_split);
    cudaError_t e = cudaSuccess;
    auto alloc = [&](void** p, size_t n) {
        if (e == cudaSuccess) e = cudaMalloc(p, n);
    };
    alloc((void**)&m->h, (size_t)d.hidden * 4);
    alloc((void**)&m->q, (size_t)qd * 4);
    alloc((void**)&m->att, (size_t)qd * 4);
    alloc((void**)&m->act, (size_t)d.ffn * 4);
    alloc((void**)&m->step, 16);
    alloc((void**)&m->rope, (size_t)d.head_dim * 4);
    alloc((void**)&m->h_prev, (size_t)d.hidden * 4);
    alloc((void**)&m->cos_dev, (size_t)d.n_layers * 4);
    alloc(&m->attn_ws, ws);
    if (e == cudaSuccess) e = cudaMemset(m->attn_ws, 0, ws);
    if (e == cudaSuccess) e = cudaMemset(m->step, 0, 16);
    if (e == cudaSuccess && d.n_resident < d.n_layers) {
        st = choose_host_path(m);
        if (st != NTX_OK) {
            free_model(m);
            return st;
        }
        const int kvd = d.n_kv_heads * d.head_dim;
        // ring slots sized for the largest of each matrix over the streamed layers
        for (int l = d.n_resident; l < d.n_layers; ++l) {
            const ntx_layer_qt& q = m->lqt[l];
            m->sz_qkv = std::max(m->sz_qkv, (size_t)(qd + 2 * kvd) * row_bytes(q.qkv, d.hidden));
            m->sz_o = std::max(m->sz_o, (size_t)d.hidden * row_bytes(q.o, qd));
            m->sz_ffn = std::max(m->sz_ffn, (size_t)d.ffn * row_bytes(q.ffn, d.hidden));
            m->sz_down = std::max(m->sz_down, (size_t)d.hidden * row_bytes(q.down, d.ffn));
        }
        m->off_qkv = 0;
        m->off_o = align256(m->sz_qkv);
        m->off_gate = m->off_o + align256(m->sz_o);
        m->off_up = m->off_gate + align256(m->sz_ffn);
        m->off_down = m->off_up + align256(m->sz_ffn);
        m->slot_bytes = m->off_down + align256(m->sz_down);
        alloc((void**)&m->ring, 2 * m->slot_bytes);
        for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&m->copy_done[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&m->slot_free[i], cudaEventDisableTiming);
        }
    }
    if (e == cudaSuccess) e = cudaEventCreate(&m->ev_start);
    if (e == cudaSuccess) e = cudaEventCreate(&m->ev_end);
    if (e != cudaSuccess) {
        const ntx_status code = (e == cudaErrorMemoryAllocation) ? NTX_ENOMEM : NTX_ECUDA;
        free_model(m);
        return fail(code, std::string("ntx_model_create: ") + cudaGetErrorString(e));
    }
    *model = m;
    return NTX_OK;
}

NTX_EXPORT ntx_status ntx_model_destroy(ntx_model* model)
{
    if (!model) return fail(NTX_EINVAL, "ntx_model_destroy: null model");
    cudaDeviceSynchronize();
    free_model(model);
    return NTX_OK;
}

namespace ntx {
namespace {

// Record what `enqueue` queues on a capture stream as an instantiated CUDA graph (*out).
template <typename Enqueue>
ntx_status record_graph(Enqueue enqueue, cudaGraphExec_t* out, const char* who)
{
    const std::string w(who);
    cudaStream_t cap;
    NTX_CUDA_TRY(cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking));
    cudaGraph_t g = nullptr;
    cudaError_t e = cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) {
        cudaStreamDestroy(cap);
        return fail(NTX_ECUDA, w + ": begin capture: " + cudaGetErrorString(e));
    }
    const ntx_status st = enqueue(cap);
    e = cudaStreamEndCapture(cap, &g);
    cudaStreamDestroy(cap);
    if (st != NTX_OK) {
        if (g) cudaGraphDestroy(g);
        return st;
    }
    if (e != cudaSuccess) return fail(NTX_ECUDA, w + ": end capture: " + cudaGetErrorString(e));
    e = cudaGraphInstantiate(out, g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) {
        *out = nullptr;
        return fail(NTX_ECUDA, w + ": instantiate: " + cudaGetErrorString(e));
    }
    return NTX_OK;
}

}  // namespace
}  // namespace ntx

NTX_EXPORT ntx_status ntx_decode_step(ntx_model* m, int32_t token, int32_t pos, float* logits, void* stream)
{
    if (!m || !logits) return fail(NTX_EINVAL, "ntx_decode_step: null pointer");
    if (m->d.n_resident != m->d.n_layers)
        return fail(NTX_EINVAL, "ntx_decode_step: model has streamed layers; use ntx_stream_layers");
    if (token < 0 || token >= m->d.vocab) return fail(NTX_EINVAL, "ntx_decode_step: token out of range");
    if (pos < 0 || pos >= m->d.max_ctx) return fail(NTX_EINVAL, "ntx_decode_step: pos out of range");
    if (!aligned(logits, 4)) return fail(NTX_EINVAL, "ntx_decode_step: logits must be 4-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    ntx_status st = set_step_launch(m->step, token, pos, m->rope, m->d.rope_theta, m->d.head_dim, s);
    if (st != NTX_OK) return st;
    if (!m->use_graph) return enqueue_resident(m, m->d.n_layers, logits, s, true);
    if (!m->graph || m->graph_logits != logits) {
        if (m->graph) {
            cudaGraphExecDestroy(m->graph);
            m->graph = nullptr;
        }
        st = record_graph([&](cudaStream_t cap) { return enqueue_resident(m, m->d.n_layers, logits, cap, true); },
                          &m->graph, "ntx_decode_step");
        if (st != NTX_OK) return st;
        m->graph_logits = logits;
    }
    NTX_CUDA_TRY(cudaGraphLaunch(m->graph, s));
    return NTX_OK;
}

namespace ntx {
namespace {

// The ring's operations on two CUDA streams: copies (cudaMemcpyAsync from the host
// pointers of the layer descriptors) on `ks`, compute on `cs`, events between them.
struct CudaRing final : ring::Ops {
    ntx_model* m;
    cudaStream_t cs, ks;
    const Lane* lanes;
    int n_lanes;
    int64_t h2d = 0;
    CudaRing(ntx_model* m_, cudaStream_t cs_, cudaStream_t ks_, const Lane* lanes_, int n_lanes_)
        : m(m_), cs(cs_), ks(ks_), lanes(lanes_), n_lanes(n_lanes_) {}

    uint8_t* slot_base(int slot) const { return m->ring + (size_t)slot * m->slot_bytes; }

    ntx_status copy_wait_slot(int slot) override
    {
        NTX_CUDA_TRY(cudaStreamWaitEvent(ks, m->slot_free[slot], 0));
        return NTX_OK;
    }
    ntx_status copy_layer(int j, int slot) override
    {
        // this layer's own matrix sizes (its formats may differ from the largest the slot holds)
        const ntx_model_desc& d = m->d;
        const ntx_layer_desc& L = m->layers[j];
        const ntx_layer_qt& q = m->lqt[j];
        const int kvd = d.n_kv_heads * d.head_dim, qd = d.n_q_heads * d.head_dim;
        const size_t b_qkv = (size_t)(qd + 2 * kvd) * row_bytes(q.qkv, d.hidden);
        const size_t b_o = (size_t)d.hidden * row_bytes(q.o, qd);
        const size_t b_ffn = (size_t)d.ffn * row_bytes(q.ffn, d.hidden);
        const size_t b_down = (size_t)d.hidden * row_bytes(q.down, d.ffn);
        uint8_t* base = slot_base(slot);
        NTX_CUDA_TRY(cudaMemcpyAsync(base + m->off_qkv, L.w_qkv, b_qkv, cudaMemcpyHostToDevice, ks));
        NTX_CUDA_TRY(cudaMemcpyAsync(base + m->off_o, L.w_o, b_o, cudaMemcpyHostToDevice, ks));
        NTX_CUDA_TRY(cudaMemcpyAsync(base + m->off_gate, L.w_gate, b_ffn, cudaMemcpyHostToDevice, ks));
        NTX_CUDA_TRY(cudaMemcpyAsync(base + m->off_up, L.w_up, b_ffn, cudaMemcpyHostToDevice, ks));
        NTX_CUDA_TRY(cudaMemcpyAsync(base + m->off_down, L.w_down, b_down, cudaMemcpyHostToDevice, ks));
        h2d += (int64_t)(b_qkv + b_o + 2 * b_ffn + b_down);
        return NTX_OK;
    }
    ntx_status copy_done(int slot) override
    {
        NTX_CUDA_TRY(cudaEventRecord(m->copy_done[slot], ks));
        return NTX_OK;
    }
    ntx_status compute_wait_copy(int slot) override
    {
        NTX_CUDA_TRY(cudaStreamWaitEvent(cs, m->copy_done[slot], 0));
        return NTX_OK;
    }
    ntx_status compute_layer(int j, int slot) override
    {
        uint8_t* base = slot_base(slot);
        const LayerW w{base + m->off_qkv, base + m->off_o, base + m->off_gate, base + m->off_up, base + m->off_down};
        // every lane goes through the layer while its matrices are in the slot: one copy
        // over the host link serves all of them
        return enqueue_layer_lanes(m, j, w, cs, false, lanes, n_lanes);
    }
    ntx_status compute_done(int slot) override
    {
        NTX_CUDA_TRY(cudaEventRecord(m->slot_free[slot], cs));
        return NTX_OK;
    }
    ntx_status before_streamed() override
    {
        return enqueue_resident(m, m->d.n_resident, nullptr, cs, lanes, n_lanes);
    }
};

}  // namespace
}  // namespace ntx

namespace ntx {
namespace {

// Queue one pass of a partly resident model over the given lanes (their step words
// already written): resident layers, then the streamed layers through the ring, each
// streamed layer copied once for all lanes; the heads when logits is not null.
ntx_status enqueue_streamed_pass(ntx_model* m, float* logits, cudaStream_t cs, cudaStream_t ks, const Lane* lanes,
                                 int n_lanes)
{
    const ntx_model_desc& d = m->d;
    ntx_status st;
    // the streamed layers that run (skipped layers are neither copied nor computed)
    std::vector<int> streamed;
    for (int j = d.n_resident; j < d.n_layers; ++j)
        if (layer_runs(m, j, nullptr)) streamed.push_back(j);
    if (!streamed.empty()) NTX_CUDA_TRY(cudaStreamWaitEvent(ks, m->ev_start, 0));
    CudaRing ops(m, cs, ks, lanes, n_lanes);
    if ((st = ring::schedule(ops, streamed.data(), (int)streamed.size(), 2)) != NTX_OK) return st;
    if (logits && (st = enqueue_heads(m, logits, cs, false, lanes, n_lanes)) != NTX_OK) return st;
    NTX_CUDA_TRY(cudaEventRecord(m->ev_end, cs));
    m->last_h2d = ops.h2d;
    return NTX_OK;
}

// One step of a partly resident model (the model's own lane); the head when logits is
// not null.
ntx_status enqueue_streamed_step(ntx_model* m, int32_t token, int32_t pos, float* logits, cudaStream_t cs,
                                 cudaStream_t ks)
{
    const ntx_model_desc& d = m->d;
    NTX_CUDA_TRY(cudaEventRecord(m->ev_start, cs));
    const ntx_status st = set_step_launch(m->step, token, pos, m->rope, d.rope_theta, d.head_dim, cs);
    if (st != NTX_OK) return st;
    const Lane ln = lane0(m);
    return enqueue_streamed_pass(m, logits, cs, ks, &ln, 1);
}

}  // namespace
}  // namespace ntx

NTX_EXPORT ntx_status ntx_stream_layers(ntx_model* m, int32_t token, int32_t pos, float* logits, void* compute,
                                        void* copy, int64_t timeout_ms)
{
    if (!m || !logits) return fail(NTX_EINVAL, "ntx_stream_layers: null pointer");
    if (token < 0 || token >= m->d.vocab) return fail(NTX_EINVAL, "ntx_stream_layers: token out of range");
    if (pos < 0 || pos >= m->d.max_ctx) return fail(NTX_EINVAL, "ntx_stream_layers: pos out of range");
    if (timeout_ms < 0) return fail(NTX_EINVAL, "ntx_stream_layers: timeout_ms must be >= 0");
    if (!aligned(logits, 4)) return fail(NTX_EINVAL, "ntx_stream_layers: logits must be 4-byte aligned");
    if (compute == copy && m->d.n_resident < m->d.n_layers)
        return fail(NTX_EINVAL, "ntx_stream_layers: compute and copy streams must differ");
    ntx_status st = enqueue_streamed_step(m, token, pos, logits, (cudaStream_t)compute, (cudaStream_t)copy);
    if (st != NTX_OK) return st;
    if (timeout_ms > 0) {
        cudaError_t qerr = cudaSuccess;
        st = ring::wait_bounded(
            [&]() -> ntx_status {
                const cudaError_t q = cudaEventQuery(m->ev_end);
                if (q == cudaSuccess) return NTX_OK;
                if (q == cudaErrorNotReady) return NTX_ETIMEOUT;
                qerr = q;
                return NTX_ECUDA;
            },
            timeout_ms);
        if (st == NTX_ETIMEOUT)
            return fail(NTX_ETIMEOUT, "ntx_stream_layers: step not finished within timeout_ms (work stays queued)");
        if (st != NTX_OK) return fail(st, std::string("ntx_stream_layers: ") + cudaGetErrorString(qerr));
    }
    return NTX_OK;
}

NTX_EXPORT ntx_status ntx_stream_stats(ntx_model* m, int64_t* h2d_bytes, float* step_ms)
{
    if (!m) return fail(NTX_EINVAL, "ntx_stream_stats: null model");
    if (h2d_bytes) *h2d_bytes = m->last_h2d;
    if (step_ms) {
        float ms = 0.f;
        NTX_CUDA_TRY(cudaEventElapsedTime(&ms, m->ev_start, m->ev_end));
        *step_ms = ms;
    }
    return NTX_OK;
}

NTX_EXPORT ntx_status ntx_model_replay_gemv(ntx_model* m, int kind, int n_launches, float* logits, void* stream)
{
    if (!m) return fail(NTX_EINVAL, "ntx_model_replay_gemv: null model");
    if (kind < NTX_GEMV_QKV || kind > NTX_GEMV_HEAD) return fail(NTX_EINVAL, "ntx_model_replay_gemv: unknown kind");
    if (n_launches < 1) return fail(NTX_EINVAL, "ntx_model_replay_gemv: n_launches must be >= 1");
    if (kind == NTX_GEMV_HEAD && (!logits || !aligned(logits, 4)))
        return fail(NTX_EINVAL, "ntx_model_replay_gemv: the LM head needs 4-byte aligned logits");
    const int nres = m->d.n_resident;
    if (kind != NTX_GEMV_HEAD && nres < 1) return fail(NTX_EINVAL, "ntx_model_replay_gemv: no resident layer");
    cudaStream_t s = (cudaStream_t)stream;
    ntx_status st = NTX_OK;
    for (int i = 0; i < n_launches && st == NTX_OK; ++i) {
        const int l = i % std::max(1, nres);
        const ntx_layer_desc& L = m->layers[l];
        switch (kind) {
        case NTX_GEMV_QKV: st = launch_qkv(m, l, L.w_qkv, s, m->pdl, lane0(m)); break;
        case NTX_GEMV_O: st = launch_o(m, l, L.w_o, s, m->pdl, lane0(m)); break;
        case NTX_GEMV_GATE_UP: st = launch_gate_up(m, l, L.w_gate, L.w_up, s, m->pdl, lane0(m)); break;
        case NTX_GEMV_DOWN: st = launch_down(m, l, L.w_down, s, m->pdl, lane0(m)); break;
        default: st = enqueue_head(m, logits, s, m->pdl, lane0(m)); break;
        }
    }
    return st;
}

NTX_EXPORT ntx_status ntx_model_set_layer_skip(ntx_model* m, const uint8_t* skip)
{
    if (!m) return fail(NTX_EINVAL, "ntx_model_set_layer_skip: null model");
    for (int l = 0; l < m->d.n_layers; ++l) m->skip[l] = skip && skip[l] ? 1 : 0;
    // the recorded step and passes hold the old set of layers: record them again on the next call
    if (m->graph) {
        cudaGraphExecDestroy(m->graph);
        m->graph = nullptr;
    }
    for (cudaGraphExec_t& g : m->vgraph) {
        if (g) cudaGraphExecDestroy(g);
        g = nullptr;
    }
    if (m->dgraph) {
        cudaGraphExecDestroy(m->dgraph);
        m->dgraph = nullptr;
    }
    return NTX_OK;
}

NTX_EXPORT ntx_status ntx_model_layer_similarity(ntx_model* m, int32_t token, int32_t pos, float* cos_out,
                                                 void* compute, void* copy)
{
    if (!m || !cos_out) return fail(NTX_EINVAL, "ntx_model_layer_similarity: null pointer");
    if (token < 0 || token >= m->d.vocab) return fail(NTX_EINVAL, "ntx_model_layer_similarity: token out of range");
    if (pos < 0 || pos >= m->d.max_ctx) return fail(NTX_EINVAL, "ntx_model_layer_similarity: pos out of range");
    const bool streamed = m->d.n_resident < m->d.n_layers;
    if (streamed && compute == copy)
        return fail(NTX_EINVAL, "ntx_model_layer_similarity: compute and copy streams must differ");
    cudaStream_t cs = (cudaStream_t)compute;
    NTX_CUDA_TRY(cudaMemsetAsync(m->cos_dev, 0, (size_t)m->d.n_layers * 4, cs));
    m->calibrating = true;
    const bool pdl = m->pdl;
    m->pdl = false;
    ntx_status st;
    if (streamed) {
        st = enqueue_streamed_step(m, token, pos, nullptr, cs, (cudaStream_t)copy);
    } else {
        st = set_step_launch(m->step, token, pos, m->rope, m->d.rope_theta, m->d.head_dim, cs);
        if (st == NTX_OK) st = enqueue_resident(m, m->d.n_layers, nullptr, cs, false);
    }
    m->calibrating = false;
    m->pdl = pdl;
    if (st != NTX_OK) return st;
    NTX_CUDA_TRY(cudaMemcpyAsync(cos_out, m->cos_dev, (size_t)m->d.n_layers * 4, cudaMemcpyDeviceToHost, cs));
    NTX_CUDA_TRY(cudaStreamSynchronize(cs));
    return NTX_OK;
}

NTX_EXPORT ntx_status ntx_plan_resident(const ntx_model_desc* desc, size_t hbm_budget, int32_t* n_resident,
                                        size_t* hbm_used)
{
    if (!n_resident) return fail(NTX_EINVAL, "ntx_plan_resident: null output pointer");
    *n_resident = 0;
    if (hbm_used) *hbm_used = 0;
    const ntx_status st = check_shapes(desc);
    if (st != NTX_OK) return st;
    // the HBM need grows with n (each resident layer adds its matrices, the ring shrinks by
    // at most one layer's worth): take the largest n that fits
    int best = -1;
    size_t used = 0;
    for (int n = 0; n <= desc->n_layers; ++n) {
        const size_t b = hbm_bytes_for(desc, n);
        if (b <= hbm_budget) {
            best = n;
            used = b;
        }
    }
    if (best < 0)
        return fail(NTX_ENOMEM, "ntx_plan_resident: even with every layer streamed the model needs " +
                                    std::to_string(hbm_bytes_for(desc, 0)) + " bytes of HBM");
    *n_resident = best;
    if (hbm_used) *hbm_used = used;
    return NTX_OK;
}

NTX_EXPORT ntx_status ntx_model_host_path(ntx_model* m, int32_t* path)
{
    if (!m || !path) return fail(NTX_EINVAL, "ntx_model_host_path: null pointer");
    *path = m->host_path;
    return NTX_OK;
}

namespace ntx {
namespace {

// The buffers of multi-token passes, allocated on first use.
ntx_status ensure_lanes(ntx_model* m)
{
    if (m->lane_h) return NTX_OK;
    const ntx_model_desc& d = m->d;
    cudaError_t e = cudaMalloc((void**)&m->lane_h, (size_t)kMaxLanes * d.hidden * 4);
    if (e == cudaSuccess) e = cudaMalloc((void**)&m->lane_step, (size_t)kMaxLanes * 16);
    if (e == cudaSuccess) e = cudaMalloc((void**)&m->lane_rope, (size_t)kMaxLanes * d.head_dim * 4);
    if (e == cudaSuccess)
        e = cudaMalloc((void**)&m->lane_act, (size_t)kMaxLanes * (2 * d.n_q_heads * d.head_dim + d.ffn) * 4);
    if (e == cudaSuccess) e = cudaMalloc((void**)&m->spec_tokens, (size_t)2 * kMaxLanes * 4);
    if (e == cudaSuccess) e = cudaMalloc((void**)&m->spec_logits, (size_t)kMaxLanes * d.vocab * 4);
    if (e != cudaSuccess) {
        cudaFree(m->lane_h);
        cudaFree(m->lane_step);
        cudaFree(m->lane_rope);
        cudaFree(m->lane_act);
        cudaFree(m->spec_tokens);
        cudaFree(m->spec_logits);
        m->lane_h = nullptr;
        m->lane_step = nullptr;
        m->lane_rope = nullptr;
        m->lane_act = nullptr;
        m->spec_tokens = nullptr;
        m->spec_logits = nullptr;
        return fail(e == cudaErrorMemoryAllocation ? NTX_ENOMEM : NTX_ECUDA,
                    std::string("multi-token pass buffers: ") + cudaGetErrorString(e));
    }
    return NTX_OK;
}

Lane lane_at(ntx_model* m, int i)
{
    const ntx_model_desc& d = m->d;
    const size_t qd = (size_t)d.n_q_heads * d.head_dim;
    float* a = m->lane_act + (size_t)i * (2 * qd + d.ffn);
    return {m->lane_h + (size_t)i * d.hidden, m->lane_step + 4 * i, m->lane_rope + (size_t)i * d.head_dim, a, a + qd,
            a + 2 * qd};
}

// One pass of the full model over n tokens at positions pos0 .. pos0 + n - 1 (token i
// from host tokens[i], or from device tokens_dev[i] when that is not null), logits of
// token i into logits + i vocab.  Resident models run on `cs` alone.
ntx_status enqueue_multi(ntx_model* m, const int32_t* tokens, const int32_t* tokens_dev, int n, int32_t pos0,
                         float* logits, cudaStream_t cs, cudaStream_t ks)
{
    const ntx_model_desc& d = m->d;
    Lane lanes[kMaxLanes];
    NTX_CUDA_TRY(cudaEventRecord(m->ev_start, cs));
    for (int i = 0; i < n; ++i) {
        lanes[i] = lane_at(m, i);
        const ntx_status st = set_step_launch(lanes[i].step, tokens ? tokens[i] : 0, pos0 + i, lanes[i].rope,
                                              d.rope_theta, d.head_dim, cs, tokens_dev ? tokens_dev + i : nullptr);
        if (st != NTX_OK) return st;
    }
    if (d.n_resident == d.n_layers) {
        // the pass body reads every token and position from the lanes' step words, so it is
        // recorded once per token count (and logits buffer) and replayed
        if (!m->use_graph) {
            const ntx_status st = enqueue_resident(m, d.n_layers, logits, cs, lanes, n);
            if (st != NTX_OK) return st;
        } else {
            if (!m->vgraph[n] || m->vgraph_logits[n] != logits) {
                if (m->vgraph[n]) {
                    cudaGraphExecDestroy(m->vgraph[n]);
                    m->vgraph[n] = nullptr;
                }
                const ntx_status st = record_graph(
                    [&](cudaStream_t cap) { return enqueue_resident(m, d.n_layers, logits, cap, lanes, n); },
                    &m->vgraph[n], "verification pass");
                if (st != NTX_OK) return st;
                m->vgraph_logits[n] = logits;
            }
            NTX_CUDA_TRY(cudaGraphLaunch(m->vgraph[n], cs));
        }
        NTX_CUDA_TRY(cudaEventRecord(m->ev_end, cs));
        return NTX_OK;
    }
    return enqueue_streamed_pass(m, logits, cs, ks, lanes, n);
}

ntx_status check_multi(ntx_model* m, int n, int32_t pos0, void* compute, void* copy, const char* who)
{
    const std::string w(who);
    if (!m) return fail(NTX_EINVAL, w + ": null model");
    if (n < 1 || n > kMaxLanes) return fail(NTX_EINVAL, w + ": between 1 and 8 tokens");
    if (pos0 < 0 || pos0 + n > m->d.max_ctx) return fail(NTX_EINVAL, w + ": positions out of range");
    if (m->d.n_resident < m->d.n_layers && compute == copy)
        return fail(NTX_EINVAL, w + ": compute and copy streams must differ");
    return ensure_lanes(m);
}

}  // namespace
}  // namespace ntx

NTX_EXPORT ntx_status ntx_verify_tokens(ntx_model* m, const int32_t* tokens, int32_t n, int32_t pos0, float* logits,
                                        void* compute, void* copy)
{
    ntx_status st = check_multi(m, n, pos0, compute, copy, "ntx_verify_tokens");
    if (st != NTX_OK) return st;
    if (!tokens || !logits || !aligned(logits, 4)) return fail(NTX_EINVAL, "ntx_verify_tokens: bad tokens / logits");
    for (int i = 0; i < n; ++i)
        if (tokens[i] < 0 || tokens[i] >= m->d.vocab) return fail(NTX_EINVAL, "ntx_verify_tokens: token out of range");
    return enqueue_multi(m, tokens, nullptr, n, pos0, logits, (cudaStream_t)compute, (cudaStream_t)copy);
}

NTX_EXPORT ntx_status ntx_speculative_step(ntx_model* m, int32_t token, int32_t pos, int32_t k,
                                           const uint8_t* draft_skip, int32_t* out_tokens, int32_t* n_out,
                                           void* compute, void* copy, int64_t timeout_ms)
{
    ntx_status st = check_multi(m, k, pos, compute, copy, "ntx_speculative_step");
    if (st != NTX_OK) return st;
    if (k < 2) return fail(NTX_EINVAL, "ntx_speculative_step: k must be at least 2");
    if (!out_tokens || !n_out) return fail(NTX_EINVAL, "ntx_speculative_step: null output pointer");
    if (token < 0 || token >= m->d.vocab) return fail(NTX_EINVAL, "ntx_speculative_step: token out of range");
    if (timeout_ms < 0) return fail(NTX_EINVAL, "ntx_speculative_step: timeout_ms must be >= 0");
    const ntx_model_desc& d = m->d;
    cudaStream_t cs = (cudaStream_t)compute, ks = (cudaStream_t)copy;
    int32_t* drafted = m->spec_tokens;              // [k]: token, then the k - 1 drafted tokens
    int32_t* predicted = m->spec_tokens + kMaxLanes;
    // the draft model: the resident layers (streamed layers left out) minus draft_skip
    std::vector<uint8_t> also(d.n_layers, 0);
    for (int l = 0; l < d.n_layers; ++l) also[l] = (l >= d.n_resident || (draft_skip && draft_skip[l])) ? 1 : 0;
    NTX_CUDA_TRY(cudaMemcpyAsync(drafted, &token, 4, cudaMemcpyHostToDevice, cs));
    const Lane ln = lane0(m);
    // the draft step's body reads its token and position from the step word: recorded once
    // per set of draft layers and replayed
    if (m->use_graph && (!m->dgraph || m->dgraph_also != also)) {
        if (m->dgraph) {
            cudaGraphExecDestroy(m->dgraph);
            m->dgraph = nullptr;
        }
        st = record_graph(
            [&](cudaStream_t cap) { return enqueue_resident(m, d.n_layers, m->spec_logits, cap, &ln, 1, also.data()); },
            &m->dgraph, "draft step");
        if (st != NTX_OK) return st;
        m->dgraph_also = also;
    }
    for (int i = 0; i + 1 < k && st == NTX_OK; ++i) {
        // draft step i: the token drafted last, at pos + i; greedy pick of the next one (the
        // step word, written by a plain launch that reads the drafted token, precedes every
        // programmatic dependent of the step, as in ntx_decode_step)
        st = set_step_launch(ln.step, 0, pos + i, ln.rope, d.rope_theta, d.head_dim, cs, drafted + i);
        if (st == NTX_OK) {
            if (m->use_graph) {
                const cudaError_t e = cudaGraphLaunch(m->dgraph, cs);
                if (e != cudaSuccess) st = fail(NTX_ECUDA, std::string("draft step: ") + cudaGetErrorString(e));
            } else {
                st = enqueue_resident(m, d.n_layers, m->spec_logits, cs, &ln, 1, also.data());
            }
        }
        if (st == NTX_OK) st = argmax_launch(m->spec_logits, d.vocab, drafted + i + 1, cs);
    }
    if (st != NTX_OK) return st;
    // one pass of the full model over the token and the drafted tokens
    if ((st = enqueue_multi(m, nullptr, drafted, k, pos, m->spec_logits, cs, ks)) != NTX_OK) return st;
    for (int i = 0; i < k; ++i)
        if ((st = argmax_launch(m->spec_logits + (size_t)i * d.vocab, d.vocab, predicted + i, cs)) != NTX_OK)
            return st;
    int32_t host[2 * kMaxLanes];
    NTX_CUDA_TRY(cudaMemcpyAsync(host, m->spec_tokens, sizeof(host), cudaMemcpyDeviceToHost, cs));
    NTX_CUDA_TRY(cudaEventRecord(m->ev_end, cs));
    st = ring::wait_bounded(
        [&]() -> ntx_status {
            const cudaError_t q = cudaEventQuery(m->ev_end);
            return q == cudaSuccess ? NTX_OK : q == cudaErrorNotReady ? NTX_ETIMEOUT : NTX_ECUDA;
        },
        timeout_ms > 0 ? timeout_ms : (int64_t)1 << 40);
    if (st == NTX_ETIMEOUT)
        return fail(NTX_ETIMEOUT, "ntx_speculative_step: not finished within timeout_ms (work stays queued)");
    if (st != NTX_OK) return fail(st, "ntx_speculative_step: a kernel failed");
    // accept the drafted tokens the full model predicts too, then its own next token
    int n = 0;
    while (n + 1 < k && host[kMaxLanes + n] == host[n + 1]) {
        out_tokens[n] = host[n + 1];
        ++n;
    }
    out_tokens[n] = host[kMaxLanes + n];
    *n_out = n + 1;
    return NTX_OK;
}

NTX_EXPORT ntx_status ntx_model_step_launches(ntx_model* m, int32_t* launches)
{
    if (!m || !launches) return fail(NTX_EINVAL, "ntx_model_step_launches: null pointer");
    int n = 0;
    for (int l = 0; l < m->d.n_layers; ++l)
        if (layer_runs(m, l, nullptr)) ++n;
    // per layer: QKV, attention, the merge of its splits, O, gate/up, down; plus the step
    // word, the embedding and the LM head
    *launches = 3 + 6 * n;
    return NTX_OK;
}
