"""Seeded synthetic inputs (models, item vectors, requests) shared by the
tests, the benchmark and the oracle.  No step of the ranking method lives
here."""
