"""CUDA graphs and the encoder side stream: replayed or overlapped steps give
the same bits as the plain eager calls.
"""
import pytest
import torch

from tests.gpu_util import pixels_to_device, tower_to_device
from vision_language_model_b200 import synth, vlm

pytestmark = pytest.mark.gpu

SIZES = [(224, 224), (112, 168), (56, 280)]


def _pipeline(layers=2, seed=3):
    cfg = vlm.preset("mistral3", layers=layers)
    tw = synth.tower_weights(seed, layers, cfg.width, cfg.mlp, cfg.patch)
    pw = synth.projector_weights(seed, cfg.width, cfg.merge, cfg.proj_out)
    return cfg, vlm.ImagePipeline(cfg, tower_to_device(tw), tower_to_device(pw), SIZES)


def _text_setup(cfg, pipe, seed=3, seq_len=2048):
    runs = [[n] for n in [(h // 28) * (w // 28) for h, w in SIZES]]
    ids = synth.text_sequences(seed, 3, seq_len, runs).reshape(-1).cuda()
    text = synth.text_embeddings(seed, ids.numel(), cfg.proj_out).cuda()
    return ids, text


def test_graph_replay_matches_eager_and_reads_live_inputs():
    cfg, pipe = _pipeline()
    ids, text0 = _text_setup(cfg, pipe)
    pix = pixels_to_device(synth.images(3, SIZES))
    text = text0.clone()
    ws = torch.empty(vlm.scatter_workspace_size(ids.numel()), dtype=torch.uint8, device="cuda")

    def step():
        pipe(pix)
        vlm.scatter(ids, pipe.embeds, text, cfg.image_token_id, workspace=ws, status=pipe.status)

    step()
    torch.cuda.synchronize()
    eager_emb, eager_text = pipe.embeds.clone(), text.clone()

    g = vlm.GraphStep(step)
    assert g.launches_per_replay > 3 * cfg.layers
    text.copy_(text0)
    g()
    torch.cuda.synchronize()
    assert vlm.status_sync(pipe.status) == vlm.OK
    assert torch.equal(pipe.embeds, eager_emb)
    assert torch.equal(text, eager_text)

    # new pixels in the same buffer: the replay must see them
    pix.copy_(pixels_to_device(synth.images(4, SIZES)))
    step()
    torch.cuda.synchronize()
    eager2 = pipe.embeds.clone()
    pix.copy_(pixels_to_device(synth.images(3, SIZES)))
    g()
    torch.cuda.synchronize()
    assert torch.equal(pipe.embeds, eager_emb)
    pix.copy_(pixels_to_device(synth.images(4, SIZES)))
    g()
    torch.cuda.synchronize()
    assert torch.equal(pipe.embeds, eager2)


def test_side_stream_overlaps_other_work_and_matches_eager():
    cfg, pipe = _pipeline()
    ids, text0 = _text_setup(cfg, pipe)
    requests = [pixels_to_device(synth.images(s, SIZES)) for s in (5, 6)]

    # eager reference: one stream, one request after the other
    ref = []
    for pix in requests:
        t = text0.clone()
        pipe(pix)
        vlm.scatter(ids, pipe.embeds, t, cfg.image_token_id, status=pipe.status)
        torch.cuda.synchronize()
        ref.append(t)

    side = vlm.EncoderSideStream(pipe)
    a = torch.randn(4096, 4096, device="cuda", dtype=torch.bfloat16)
    busy = torch.empty_like(a)
    outs = []
    for pix in requests:
        side.submit(pix)
        for _ in range(8):  # other work on the caller's stream while the encoder runs
            torch.matmul(a, a, out=busy)
        t = text0.clone()
        side.scatter(ids, t)
        outs.append(t)
    torch.cuda.synchronize()
    assert vlm.status_sync(pipe.status) == vlm.OK
    for got, want in zip(outs, ref):
        assert torch.equal(got, want)


def test_host_fed_steps_match_eager():
    """Inputs from pinned host memory, copies overlapped on a copy stream:
    the host result equals the eager single-stream result, run after run."""
    cfg, pipe = _pipeline()
    ids, text0 = _text_setup(cfg, pipe)
    results = []
    for seed in (8, 9):
        pix_host = torch.cat([im.reshape(-1) for im in synth.images(seed, SIZES)]).pin_memory()
        ids_host = ids.cpu().pin_memory()
        t = text0.clone()
        pipe(pix_host.cuda())
        vlm.scatter(ids, pipe.embeds, t, cfg.image_token_id, status=pipe.status)
        torch.cuda.synchronize()

        def step(inputs, result):
            emb = pipe(inputs[0])
            vlm.scatter(inputs[1], emb, result, cfg.image_token_id, status=pipe.status)

        fed = vlm.HostFedSteps(step, [pix_host.cuda(), ids], text0)
        out_host = torch.empty(text0.shape, dtype=text0.dtype, pin_memory=True)
        fed.run([pix_host, ids_host], out_host, 3)
        torch.cuda.synchronize()
        assert vlm.status_sync(pipe.status) == vlm.OK
        assert torch.equal(out_host, t.cpu())
        results.append(out_host.clone())
    assert not torch.equal(results[0], results[1])


def test_side_stream_runs_concurrently_and_matches_oracle():
    """NEXT row 1 (the encoder on its own stream): two requests of one 896x1344
    image (2 layers) submitted to the side stream while bf16 GEMMs run on the
    caller's stream. The encoder's interval (side-stream events around each
    request) and the other work's interval (caller-stream events) overlap in
    time, and every scattered row equals the oracle's embedding to tolerance,
    the other rows staying bit-identical."""
    import numpy as np
    from oracle import vlm_oracle as O
    from tests.gpu_util import compare, to_oracle

    sizes = [(896, 1344)]
    cfg = vlm.preset("mistral3", layers=2)
    tw = synth.tower_weights(13, 2, cfg.width, cfg.mlp, cfg.patch)
    pw = synth.projector_weights(13, cfg.width, cfg.merge, cfg.proj_out)
    pipe = vlm.ImagePipeline(cfg, tower_to_device(tw), tower_to_device(pw), sizes)
    ids = synth.text_sequences(13, 1, 4096, [[1536]]).reshape(-1).cuda()
    text0 = synth.text_embeddings(13, ids.numel(), cfg.proj_out).cuda()
    images = [synth.images(s, sizes) for s in (14, 15)]
    requests = [pixels_to_device(im) for im in images]

    side = vlm.EncoderSideStream(pipe)
    main = torch.cuda.current_stream()
    a = torch.randn(4096, 4096, device="cuda", dtype=torch.bfloat16)
    busy = torch.empty_like(a)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    ref = ev()
    ref.record(main)
    outs, spans = [], []
    for pix in requests:
        e0 = ev()
        e0.record(main)  # the side stream waits on the caller's stream, so this precedes its work
        side.ready = ev()  # a timing event, one per request, for the check below
        side.submit(pix)
        m0, m1 = ev(), ev()
        m0.record(main)
        for _ in range(12):  # other work on the caller's stream while the encoder runs
            torch.matmul(a, a, out=busy)
        m1.record(main)
        t = text0.clone()
        side.scatter(ids, t)
        outs.append(t)
        spans.append((e0, side.ready, m0, m1))
    torch.cuda.synchronize()
    assert vlm.status_sync(pipe.status) == vlm.OK
    for e0, ready, m0, m1 in spans:
        enc = (ref.elapsed_time(e0), ref.elapsed_time(ready))
        other = (ref.elapsed_time(m0), ref.elapsed_time(m1))
        assert enc[0] < other[1] and other[0] < enc[1], (enc, other)  # the two intervals overlap
    mask = (ids == 10).cpu()
    for got, im in zip(outs, images):
        _, ref_emb = O.encode_merge_project([x.double().numpy() for x in im], to_oracle(tw), to_oracle(pw),
                                           dict(O.MISTRAL3, layers=2))
        compare(got[mask.cuda()], ref_emb, what="side-stream scattered rows")
        assert torch.equal(got[~mask.cuda()].view(torch.int16), text0[~mask.cuda()].view(torch.int16))
    assert not np.array_equal(outs[0].cpu().float().numpy(), outs[1].cpu().float().numpy())


@pytest.mark.parametrize("kind", ["bf16", "fp8", "nvfp4"])
def test_sm_budget_gives_the_same_bits(kind):
    """vlm_config.sm_budget only changes how many SMs the persistent GEMMs hold
    and splits attention into successive grids of at most 2 CTAs per budgeted
    SM: every tile computes the same thing, so the results are bit-identical for
    every budget (2 SMs, 40, 95, and above the SM count)."""
    layers, seed = 2, 5
    tw = tower_to_device(synth.tower_weights(seed, layers, 1024, 4096, 14))
    pw = tower_to_device(synth.projector_weights(seed, 1024, 2, 5120))
    extra = {"fp8": dict(fp8_act_scales=synth.fp8_act_scales(layers)),
             "nvfp4": dict(nvfp4_act_scales=synth.nvfp4_act_scales(layers))}.get(kind, {})
    pix = pixels_to_device(synth.images(seed, SIZES))
    outs = []
    for budget in (0, 2, 40, 95, 100000):
        cfg = vlm.preset("mistral3", layers=layers, sm_budget=budget)
        pipe = vlm.ImagePipeline(cfg, tw, pw, SIZES, **extra)
        before = vlm.launch_count()
        pipe(pix)
        launches = vlm.launch_count() - before
        assert vlm.status_sync(pipe.status) == vlm.OK
        outs.append((budget, launches, pipe.tower_out.clone(), pipe.embeds.clone()))
    base = outs[0]
    qtiles = sum(((h // 14) * (w // 14) + 127) // 128 for h, w in SIZES)
    for budget, launches, tower, emb in outs[1:]:
        assert torch.equal(tower, base[2]), budget
        assert torch.equal(emb, base[3]), budget
        if 0 < budget < torch.cuda.get_device_properties(0).multi_processor_count:
            chunk = max(1, 2 * budget // 16)
            assert launches == base[1] + layers * (-(-qtiles // chunk) - 1), (budget, launches, base[1])
        else:
            assert launches == base[1]


def test_fused_scatter_under_graph_replay_and_sm_budgets():
    """ImagePipeline.embed_into (the scatter fused into the projector's last
    linear) replayed as one CUDA graph, and run with the encoder confined to 2
    and 40 SMs, writes the same rows as the eager separate calls."""
    cfg, pipe = _pipeline()
    ids, text0 = _text_setup(cfg, pipe)
    pix = pixels_to_device(synth.images(3, SIZES))
    ref = text0.clone()
    vlm.scatter(ids, pipe(pix), ref, cfg.image_token_id, status=pipe.status)
    text = text0.clone()
    g = vlm.GraphStep(lambda: pipe.embed_into(pix, ids, text))  # one eager call first, then the capture
    text.copy_(text0)
    g()
    torch.cuda.synchronize()
    assert vlm.status_sync(pipe.status) == vlm.OK
    assert torch.equal(text, ref)
    tw = tower_to_device(synth.tower_weights(3, cfg.layers, cfg.width, cfg.mlp, cfg.patch))
    pw = tower_to_device(synth.projector_weights(3, cfg.width, cfg.merge, cfg.proj_out))
    for budget in (2, 40):
        pb = vlm.ImagePipeline(vlm.preset("mistral3", layers=cfg.layers, sm_budget=budget), tw, pw, SIZES)
        t = text0.clone()
        pb.embed_into(pix, ids, t)
        assert vlm.status_sync(pb.status) == vlm.OK
        assert torch.equal(t, ref), budget
