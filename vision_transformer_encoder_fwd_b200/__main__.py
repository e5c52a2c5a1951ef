"""Run one synthetic workload through the library and print what it produced and how long it
took (CUDA events around each call, after warm-up).

    python -m vision_transformer_encoder_fwd_b200 forward [--workload vitl16_1024_b8] [--reps N]
    python -m vision_transformer_encoder_fwd_b200 seg     [--mode slide|whole] [--head] [--reps N]
    python -m vision_transformer_encoder_fwd_b200 dense   [--reps N]

forward: vit_forward on one of the seeded workloads (descriptor + patch tokens).
seg:     vit_seg_zero_shot on one 512 x 1024 image with 150 seeded class vectors (ViT-L/16,
         windows of 384 at stride 192 in slide mode), optionally with the dino.txt head.
dense:   vit_forward_dense (encoder + projector P4 + task head, 19 classes) on ViT-S/14 at 518,
         batch 8.
Weights and inputs are the seeded synthetic ones of the test suite; nothing is trained.
"""
import argparse
import os
import sys

import torch


def _timed(fn, reps, warmup=2):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        out = fn()
    e1.record()
    torch.cuda.synchronize()
    return out, e0.elapsed_time(e1) / reps


def main(argv=None) -> int:
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synthetic as S
    import vision_transformer_encoder_fwd_b200 as V

    ap = argparse.ArgumentParser(prog="python -m vision_transformer_encoder_fwd_b200")
    ap.add_argument("what", choices=["forward", "seg", "dense"])
    ap.add_argument("--workload", default="vitl16_1024_b8", choices=sorted(S.WORKLOADS))
    ap.add_argument("--mode", default="slide", choices=["slide", "whole"])
    ap.add_argument("--head", action="store_true", help="seg: attach the dino.txt vision head")
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("needs a CUDA device")

    if args.what == "forward":
        spec, w, im = S.make_workload(args.workload)
        enc = V.VitEncoder(spec, w, max_batch=im.shape[0])
        x = im.cuda()
        outs, ms = _timed(lambda: enc.forward(x, desc=True, patch=True), args.reps)
        enc.poll()
        print(f"{args.workload}: {ms:.3f} ms per forward, {im.shape[0] / ms * 1e3:.1f} images/s; "
              f"descriptor {tuple(outs['desc'].shape)}, patch tokens {tuple(outs['patch_tokens'].shape)}, "
              f"{enc.last_launch_count()} launches")
    elif args.what == "seg":
        spec, w, im = S.make_workload("vitl16_slide_512x1024")
        enc = V.VitEncoder(spec, w, max_batch=10)
        if args.head:
            enc.set_text_head(S.make_head_weights(spec, S.HEAD_SEED))
        text = S.make_text_feats(S.SLIDE_CLASSES, spec.dim).cuda()
        x = im[0].cuda()
        mode = V.VIT_SEG_SLIDE if args.mode == "slide" else V.VIT_SEG_WHOLE
        (probs, labels), ms = _timed(
            lambda: enc.seg(x, text, mode=mode, side=S.SLIDE_SIDE, stride=S.SLIDE_STRIDE), args.reps)
        enc.poll()
        print(f"zero-shot {args.mode}{' + dino.txt head' if args.head else ''}: {ms:.3f} ms per image; "
              f"scores {tuple(probs.shape)}, labels {tuple(labels.shape)}, {enc.last_launch_count()} launches")
    else:
        spec, w, im = S.make_workload("vits14_518_b8_taps")
        enc = V.VitEncoder(spec, w, max_batch=im.shape[0])
        enc.set_dense_head(S.make_dense_head_weights(spec, S.DENSE_SEED))
        x = im.cuda()
        (logits, _), ms = _timed(lambda: enc.forward_dense(x), args.reps)
        enc.poll()
        print(f"dense head: {ms:.3f} ms per batch of {im.shape[0]}; logits {tuple(logits.shape)}, "
              f"{enc.last_launch_count()} launches")
    enc.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
