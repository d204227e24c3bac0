"""B200-native audio-encoder forward (MOSS-Audio / MOSS-Transcribe AuT tower).

The compute lives in ``libmoss_enc.so`` (hand-written sm_100a CUDA behind a
C ABI, declared in ``include/moss_enc.h``).  ``audio_encoder_b200.binding``
marshals arguments to it; ``audio_encoder_b200.synth`` makes seeded inputs.
"""
__all__ = ["binding", "synth", "build"]
