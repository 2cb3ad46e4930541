"""Parity of the image-token bridge (merge of aligner tokens and sentinels into the text
embeddings, image-span visibility of the attention mask) with the oracle, through the C ABI.

Both calls are copies, so the bar is bit-exact: the merged embeddings and the mask are compared
as raw bits.  Layouts that do not fit the images must be reported as DSV4V_ERR_LAYOUT."""
import numpy as np
import pytest
import torch

from oracle import dsv4v_oracle as O
from vision_transformer_encoder_dsv4v_b200 import dsv4v as A
from vision_transformer_encoder_dsv4v_b200 import synth

pytestmark = pytest.mark.gpu

BIG = dict(vision_dim=1024, n_heads=16, mlp_hidden=2816, downsample_ratio=2, llm_dim=4096, n_layers=1)


def cfg_of(dtype=A.DSV4V_BF16, llm_dim=4096, r=2):
    if dtype == A.DSV4V_BF16:
        return A.make_config(1024, 16, 2816, r, llm_dim, 1, 1e-6, 10000.0, A.DSV4V_BF16)
    return A.make_config(64, 4, 128, r, llm_dim, 1, 1e-6, 10000.0, A.DSV4V_F32)


def tokens_per_image(grids, r):
    return [-(-h // r) * -(-w // r) for h, w in grids]


def random_bits(shape, dtype, seed):
    """Random raw storage: int16 bit patterns for bf16, float32 normals for f32 (as int32 bits)."""
    rng = np.random.default_rng(seed)
    if dtype == A.DSV4V_BF16:
        return synth.bf16_bits(rng.standard_normal(shape, dtype=np.float32)).view(np.int16)
    return rng.standard_normal(shape, dtype=np.float32).view(np.int32)


def to_dev(bits, dtype):
    t = torch.from_numpy(np.ascontiguousarray(bits))
    t = t.view(torch.bfloat16) if dtype == A.DSV4V_BF16 else t.view(torch.float32)
    return t.cuda()


def raw(t):
    return t.cpu().view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).numpy()


def bridge_ws(types):
    return torch.empty(A.dsv4v_bridge_workspace_size(types.size), dtype=torch.uint8, device="cuda")


def run_merge(cfg, grids, types, embeds_bits, tok_bits, sent_bits, dtype):
    b = A.BatchRef(grids)
    embeds = to_dev(embeds_bits, dtype)
    ws = torch.empty(A.dsv4v_bridge_workspace_size(types.size), dtype=torch.uint8, device="cuda")
    A.dsv4v_merge_image_embeddings(cfg, b, torch.from_numpy(types).cuda(), to_dev(tok_bits, dtype),
                                   to_dev(sent_bits, dtype), embeds, ws)
    return embeds, A.dsv4v_device_error()


MERGE_CASES = {
    # grids, n_seqs, seq_len, pad_every, max_gap: several 256-position chunks and a ragged tail
    "ragged4": ([(27, 37), (37, 27), (10, 78), (112, 7)], 2, 700, 2, 40),
    "mixed": ([(3, 5), (1, 1), (64, 64), (9, 14)], 3, 1201, 3, 40),
    "tiny": ([(1, 1)], 1, 5, 0, 1),
    "one_chunk_exact": ([(28, 28)], 1, 256, 1, 40),
    "many_images": ([(1 + i % 7, 2 + i % 5) for i in range(300)], 4, 1600, 5, 8),
    # 72,003 positions: 282 chunks, long text gaps (chunks of text only)
    "long_stream": ([(40 + i % 9, 30 + i % 13) for i in range(40)], 3, 24001, 3, 400),
}


# bf16 rows of 4096 (16 column slices) and of 1024 (4 slices); f32 rows of 132 (one slice of 33
# vectors, not a divisor of the CTA's 256 threads)
@pytest.mark.parametrize("name", list(MERGE_CASES))
@pytest.mark.parametrize("dtype,llm_dim", [(A.DSV4V_BF16, 4096), (A.DSV4V_BF16, 1024), (A.DSV4V_F32, 132)])
def test_merge_image_embeddings_bit_exact(name, dtype, llm_dim):
    grids, n_seqs, seq_len, pad_every, max_gap = MERGE_CASES[name]
    cfg = cfg_of(dtype, llm_dim)
    per = tokens_per_image(grids, 2)
    types = synth.place_spans([O.image_layout(h, w, 2) for h, w in grids], n_seqs, seq_len, seed=len(grids),
                              max_gap=max_gap, pad_every=pad_every, balance=True)
    emb = random_bits((n_seqs, seq_len, llm_dim), dtype, 1)
    tok = random_bits((sum(per), llm_dim), dtype, 2)
    sent = random_bits((4, llm_dim), dtype, 3)
    got, err = run_merge(cfg, grids, types, emb, tok, sent, dtype)
    assert err == 0
    want = O.merge_image_embeddings(emb, types, tok, sent, per)
    np.testing.assert_array_equal(raw(got), want)


@pytest.mark.parametrize("mutate", ["drop_feature", "extra_feature", "open_span", "stray_pad", "nested_start",
                                    "bad_code", "few_images", "span_across_sequences", "text_in_span"])
def test_merge_image_embeddings_reports_layout_errors(mutate):
    grids = [(3, 5), (1, 1), (4, 4)]
    per = tokens_per_image(grids, 2)
    types = synth.place_spans([O.image_layout(h, w, 2) for h, w in grids], 2, 40, seed=7, max_gap=4, balance=True)
    t = types.copy()
    if mutate == "drop_feature":
        t.reshape(-1)[np.flatnonzero(t.reshape(-1) == O.TOK_IMAGE)[0]] = O.TOK_PAD
    elif mutate == "extra_feature":
        t.reshape(-1)[np.flatnonzero(t.reshape(-1) == O.TOK_NEWLINE)[0]] = O.TOK_IMAGE
    elif mutate == "open_span":
        t.reshape(-1)[np.flatnonzero(t.reshape(-1) == O.TOK_END)[-1]] = O.TOK_NEWLINE
    elif mutate == "stray_pad":
        t.reshape(-1)[np.flatnonzero(t.reshape(-1) == O.TOK_TEXT)[-1]] = O.TOK_PAD
    elif mutate == "nested_start":
        t.reshape(-1)[np.flatnonzero(t.reshape(-1) == O.TOK_IMAGE)[0]] = O.TOK_START
    elif mutate == "bad_code":
        t[0, 0] = 9
    elif mutate == "few_images":
        grids = grids + [(2, 2)]
        per = per + [1]
    elif mutate == "text_in_span":
        t.reshape(-1)[np.flatnonzero(t.reshape(-1) == O.TOK_NEWLINE)[0]] = O.TOK_TEXT
    elif mutate == "span_across_sequences":
        # the first sequence ends inside an open span that the second closes
        t = np.full((2, 8), -1, np.int32)
        t[0, 5:8] = [O.TOK_START, O.TOK_IMAGE, O.TOK_NEWLINE]
        t[1, 0:1] = [O.TOK_END]
        grids, per = [(1, 1)], [1]
    with pytest.raises(ValueError):
        O.merge_image_embeddings(np.zeros(t.shape + (1,)), t, np.zeros((sum(per), 1)), np.zeros((4, 1)), per)
    cfg = cfg_of()
    emb = random_bits(t.shape + (4096,), A.DSV4V_BF16, 4)
    _, err = run_merge(cfg, grids, t, emb, random_bits((sum(per), 4096), A.DSV4V_BF16, 5),
                       random_bits((4, 4096), A.DSV4V_BF16, 6), A.DSV4V_BF16)
    assert err == A.DSV4V_ERR_LAYOUT
    assert A.dsv4v_device_error() == 0  # the record was cleared


def visibility_case(n_seqs, seq_len, grids, seed, pad_every=0, max_gap=40):
    return synth.place_spans([O.image_layout(h, w, 2) for h, w in grids], n_seqs, seq_len, seed=seed,
                             max_gap=max_gap, pad_every=pad_every, balance=True)


@pytest.mark.parametrize("elem", [4, 2])
@pytest.mark.parametrize("case", ["short", "long_spans", "edges"])
def test_image_visibility_bit_exact(elem, case):
    if case == "short":
        types = visibility_case(3, 29, [(1, 1), (3, 5), (2, 2)], seed=11, max_gap=4)
    elif case == "long_spans":
        types = visibility_case(2, 600, [(28, 28), (27, 37), (9, 14)], seed=12, pad_every=2)
    else:
        # spans touching both ends of a sequence, back-to-back spans, a sequence of text only
        lay = O.image_layout(3, 5, 2)
        n = 2 * len(lay) + 3
        types = np.full((3, n), -1, np.int32)
        types[0, :len(lay)] = lay
        types[0, len(lay):2 * len(lay)] = lay
        types[1, n - len(lay):] = lay
    rng = np.random.default_rng(13)
    m = rng.standard_normal(types.shape + (types.shape[1],)).astype(np.float32)
    if elem == 2:
        m = synth.bf16_to_f32(synth.bf16_bits(m))
    mask = torch.from_numpy(m).cuda()
    if elem == 2:
        mask = mask.to(torch.bfloat16)
    A.dsv4v_image_visibility(torch.from_numpy(types).cuda(), mask, bridge_ws(types))
    assert A.dsv4v_device_error() == 0
    want = O.image_visibility(m.astype(np.float64), types)
    got = mask.float().cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(got, want)
    assert not np.signbit(got[want == 0]).any()  # +0 written, not -0


@pytest.mark.parametrize("bad", ["never_closed", "text_in_span", "end_first", "bad_code"])
def test_image_visibility_reports_layout_errors(bad):
    types = np.full((1, 70), -1, np.int32)
    if bad == "never_closed":
        types[0, 3:6] = [O.TOK_START, O.TOK_IMAGE, O.TOK_NEWLINE]
    elif bad == "text_in_span":  # text 40 positions after the start: found past the first warp
        types[0, 3:50] = O.TOK_IMAGE
        types[0, 3], types[0, 43], types[0, 49] = O.TOK_START, O.TOK_TEXT, O.TOK_END
    elif bad == "end_first":
        types[0, 3:6] = [O.TOK_END, O.TOK_IMAGE, O.TOK_START]
    else:
        types[0, 3:6] = [O.TOK_START, 6, O.TOK_END]
    with pytest.raises(ValueError):
        O.image_spans(types[0])
    mask = torch.zeros(1, 70, 70, device="cuda")
    A.dsv4v_image_visibility(torch.from_numpy(types).cuda(), mask, bridge_ws(types))
    assert A.dsv4v_device_error() == A.DSV4V_ERR_LAYOUT


def test_bridge_full_size_stream():
    # the 16-image high-resolution batch (4096-wide tokens) laid out in 4 sequences of 8192, the
    # size the benchmark times; merged rows bit-exact everywhere, mask rows sampled
    wl = synth.workload(5)
    grids = wl.grids
    per = tokens_per_image(grids, 2)
    types = synth.place_spans([O.image_layout(h, w, 2) for h, w in grids], 4, 8192, seed=21, pad_every=4,
                              balance=True)
    emb = random_bits((4, 8192, 4096), A.DSV4V_BF16, 22)
    tok = random_bits((sum(per), 4096), A.DSV4V_BF16, 23)
    sent = random_bits((4, 4096), A.DSV4V_BF16, 24)
    got, err = run_merge(cfg_of(), grids, types, emb, tok, sent, A.DSV4V_BF16)
    assert err == 0
    np.testing.assert_array_equal(raw(got), O.merge_image_embeddings(emb, types, tok, sent, per))
    del got
    mask = torch.full((4, 8192, 8192), float("-inf"), device="cuda")
    A.dsv4v_image_visibility(torch.from_numpy(types).cuda(), mask, bridge_ws(types))
    assert A.dsv4v_device_error() == 0
    rng = np.random.default_rng(25)
    pseudo = np.argwhere(types != O.TOK_TEXT)
    rows = np.concatenate([pseudo[rng.choice(len(pseudo), 96, replace=False)],
                           np.argwhere(types == O.TOK_TEXT)[rng.choice(int((types == -1).sum()), 32, replace=False)]])
    spans = [O.image_spans(types[b]) for b in range(4)]
    for b, i in rows:
        want = np.full(8192, -np.inf)
        for a, e in spans[b]:
            if a <= i <= e:
                want[a:e + 1] = 0.0
        np.testing.assert_array_equal(mask[b, i].cpu().numpy(), want)
