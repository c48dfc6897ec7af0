"""Plain, slow, float64 CPU oracle of the tiled distance-map sampler's hot path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or runs
anything here: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may.  It shares no code with the CUDA library and imports
nothing from the package; both sides take their inputs from :mod:`synth`.

What it computes, in the order of the method (ParaChromo paper,
mdpi.com/2079-9292/15/13/2750):

  schedule       -- linear-beta alphas-bar and the DDIM step coefficients
                    (§4.1, §5.1.1: reduced-step DDIM; Song et al., ref. [7])
  philox/noise   -- counter-based Philox4x32-10 normals keyed by
                    (seed, stream, step, sample, position)  [reading]
  ddim           -- stand-in eps, classifier-free guidance (ref. [15]), DDIM
                    update, the whole reverse run with periodic projection
  seam           -- overlap-consistency projection (§4.3.2, Algorithm 1) and
                    seam discrepancy (§5.5, Eq. 6)
  mds            -- classical MDS (the distance-geometry initialisation of
                    §3.1) and pairwise-distance reconstruction

and, beyond that path:

  schedule       -- the cosine alphas-bar table (§4.3.2 names a cosine
                    schedule; Nichol & Dhariwal 2021)
  ddim           -- the DDPM ancestral step (§5.1.2), written separately
  drift          -- the non-overlap drift of a synchronisation sweep (§5.7)
  stitch         -- Kabsch stitching of tile coordinates (§4.3.2, §5.5 Fig. 4)
  refine         -- SMACOF coordinate refinement (§3.1: "followed by
                    coordinate refinement")  [reading]

Every function is float64 and follows the definition or the algorithm's steps
as written; readings of passages that the pages leave open are stated in each
function.  Parity status: every function here is pinned by a CPU test against
something other than itself (library routines, closed forms, brute force,
invariants).  The distribution of generated maps versus a trained model is
parity unpinned (no trained model exists here).
"""
