"""DeltaKV hot path for B200 (sm_100a): residual KV-cache compression and decode attention over the
compressed, paged cache.  ``deltakv`` is the thin ctypes binding of ``libdeltakv.so``; ``synth`` draws
seeded synthetic inputs."""
__version__ = "0.1.0"
