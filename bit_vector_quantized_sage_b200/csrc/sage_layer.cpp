// Host side of the fused decoder layer: validates the shapes and describes
// the four dependent stages (q|k|v, o, gate|up, down) with their fused
// prologues and epilogue to the packed GEMV engine, which runs them in one
// launch.  The operations are those of include/sage.h (RMSNorm, attention over
// one cached position, residual add, SiLU * up), fused with the ESG
// permutation gather as Sec. 3.5 of the SAGE paper describes.
#include <vector>

#include "sage_engine.h"

namespace sage {
namespace {

struct LayerPlan {
    EngineJobSpec j0[3], j1[1], j2[2], j3[1];
    EngineStageSpec st[4];
};

int check_layer(const sage_decoder_layer* L, int M) {
    if (!L) return SAGE_ERR_INVALID_ARGUMENT;
    const sage_matrix* mats[7] = {&L->q, &L->k, &L->v, &L->o, &L->gate, &L->up, &L->down};
    for (const sage_matrix* A : mats) {
        const int rc = check_matrix(A);
        if (rc) return rc;
    }
    if (!L->attn_norm || !L->mlp_norm || !(L->eps >= 0.f)) return SAGE_ERR_INVALID_ARGUMENT;
    if (!aligned16(L->attn_norm) || !aligned16(L->mlp_norm)) return SAGE_ERR_MISALIGNED;
    if (M < 1 || M > 8) return SAGE_ERR_UNSUPPORTED;
    const int H = L->q.d_in;
    if (L->k.d_in != H || L->v.d_in != H || L->gate.d_in != H || L->up.d_in != H || L->o.d_out != H ||
        L->down.d_out != H)
        return SAGE_ERR_UNSUPPORTED;
    if (L->n_heads < 1 || L->n_kv_heads < 1 || L->head_dim < 1 || L->n_heads % L->n_kv_heads)
        return SAGE_ERR_UNSUPPORTED;
    if (L->q.d_out != L->n_heads * L->head_dim || L->o.d_in != L->q.d_out) return SAGE_ERR_UNSUPPORTED;
    if (L->k.d_out != L->n_kv_heads * L->head_dim || L->v.d_out != L->k.d_out) return SAGE_ERR_UNSUPPORTED;
    if (L->up.d_out != L->gate.d_out || L->down.d_in != L->gate.d_out) return SAGE_ERR_UNSUPPORTED;
    return SAGE_OK;
}

void make_plan(const sage_decoder_layer* L, const uint16_t* h, const sage_decoder_outputs* out, LayerPlan& P) {
    const int H = L->q.d_in;
    P.j0[0] = {L->q, nullptr, out ? out->q : nullptr};
    P.j0[1] = {L->k, nullptr, out ? out->k : nullptr};
    P.j0[2] = {L->v, nullptr, out ? out->v : nullptr};
    P.j1[0] = {L->o, nullptr, out ? out->o : nullptr};
    P.j2[0] = {L->gate, nullptr, out ? out->gate : nullptr};
    P.j2[1] = {L->up, nullptr, out ? out->up : nullptr};
    P.j3[0] = {L->down, nullptr, out ? out->down : nullptr};
    for (auto& s : P.st) s = EngineStageSpec{};
    // stage 1: RMSNorm(h) -> q | k | v
    P.st[0].jobs = P.j0; P.st[0].n_jobs = 3;
    P.st[0].stage.pro = kProRmsNorm;
    P.st[0].stage.pa = h; P.st[0].stage.pg = L->attn_norm; P.st[0].stage.pro_dim = H; P.st[0].stage.eps = L->eps;
    // stage 2: attention over one position (reads v) -> o
    P.st[1].jobs = P.j1; P.st[1].n_jobs = 1;
    P.st[1].stage.wait = 1;
    P.st[1].stage.pro = kProGqa;
    P.st[1].stage.pa = out ? out->v : nullptr; P.st[1].stage.pro_dim = L->v.d_out;
    P.st[1].stage.gqa_hd = L->head_dim; P.st[1].stage.gqa_grp = L->n_heads / L->n_kv_heads;
    // stage 3: residual + RMSNorm (reads o) -> gate | up
    P.st[2].jobs = P.j2; P.st[2].n_jobs = 2;
    P.st[2].stage.wait = 1;
    P.st[2].stage.pro = kProResidRmsNorm;
    P.st[2].stage.pa = h; P.st[2].stage.pb = out ? out->o : nullptr; P.st[2].stage.pg = L->mlp_norm;
    P.st[2].stage.pro_dim = H; P.st[2].stage.eps = L->eps;
    // stage 4: SiLU(gate) * up -> down, and the residual stream out
    P.st[3].jobs = P.j3; P.st[3].n_jobs = 1;
    P.st[3].stage.wait = 1;
    P.st[3].stage.pro = kProSiluMul;
    P.st[3].stage.pa = out ? out->gate : nullptr; P.st[3].stage.pb = out ? out->up : nullptr;
    P.st[3].stage.pro_dim = L->gate.d_out;
    P.st[3].stage.epi = kEpiResidual;
    P.st[3].stage.ea = h; P.st[3].stage.eb = out ? out->o : nullptr; P.st[3].stage.eo = out ? out->h_out : nullptr;
}

}  // namespace
}  // namespace sage

using namespace sage;

extern "C" int sage_decoder_layer_workspace_size(const sage_decoder_layer* L, int M, size_t* bytes) {
    if (!bytes) return SAGE_ERR_INVALID_ARGUMENT;
    const int rc = check_layer(L, M);
    if (rc) return rc;
    LayerPlan P;
    make_plan(L, nullptr, nullptr, P);
    *bytes = engine_workspace_bytes(P.st, 4);
    return SAGE_OK;
}

extern "C" int sage_decoder_layer_forward(const sage_decoder_layer* L, const uint16_t* h, int M,
                                          const sage_decoder_outputs* out, void* ws, size_t ws_bytes,
                                          sage_stream_t stream) {
    int rc = check_layer(L, M);
    if (rc) return rc;
    if (!h || !out || !ws) return SAGE_ERR_INVALID_ARGUMENT;
    const uint16_t* ptrs[9] = {h, out->q, out->k, out->v, out->o, out->gate, out->up, out->down, out->h_out};
    for (const uint16_t* p : ptrs) {
        if (!p) return SAGE_ERR_INVALID_ARGUMENT;
        if (!aligned16(p)) return SAGE_ERR_MISALIGNED;
    }
    LayerPlan P;
    make_plan(L, h, out, P);
    if (ws_bytes < engine_workspace_bytes(P.st, 4)) return SAGE_ERR_WORKSPACE;
    return launch_engine(P.st, 4, M, ws, ws_bytes, stream);
}
